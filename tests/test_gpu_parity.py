"""GPU parity: every stage of the CUDA path against the float64 oracle.

Inputs are the seeded synthetic workloads of hils_synth (at the sizes named in each
test), copied to the GPU; the oracle reads the very same stored bits. Bars:
  * top-K lists and counts: bit-exact (the oracle ranks by its float64 score, lower
    chunk index first on ties; lists are in ascending chunk index);
  * float outputs: bf16 max-abs <= 2e-2 and relative L2 <= 1e-2, float32 1e-4;
    Bsum (float32) within 1e-4; select scores within 1e-5 + 2e-6 |s|.
Attend stages are checked with the oracle fed the GPU's own selection, so a
selection difference can never hide inside an output check.
"""

import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_b200 as hils
from hils_synth import WORKLOADS, make_decode, make_prefill
from hils_testutil import BSUM_ATOL, assert_close, assert_same_selection, host, scores_close

pytestmark = pytest.mark.gpu


def P(w, **kw):
    return hils.Params(B=w.B, H=w.H, d=w.d, K=kw.pop("K", w.K), W=kw.pop("W", w.W), dtype=w.dtype, H_kv=w.Hk,
                       **kw)


def gpu_summarize(w, K, LQ, N=None):
    n = K.shape[2] if N is None else N
    C = n // 64
    Ksum = torch.empty(w.B, w.H, C, w.d, dtype=w.dtype, device=K.device)
    Bsum = torch.empty(w.B, w.H, C, dtype=torch.float32, device=K.device)
    hils.hils_summarize(P(w), K, LQ, Ksum, Bsum, N=n)
    return Ksum, Bsum


def gpu_select(w, Qcal, Ksum, Bsum, qpos=None, K=None):
    k = w.K if K is None else K
    p = P(w, K=k)
    B, H, Lq, Hk = Qcal.shape[0], Qcal.shape[1], Qcal.shape[2], w.Hkv
    idx = torch.full((B, Hk, Lq, k), 7777, dtype=torch.int32, device=Qcal.device)
    score = torch.full((B, H, Lq, k), 7777.0, dtype=torch.float32, device=Qcal.device)
    nsel = torch.full((B, Hk, Lq), 7777, dtype=torch.int32, device=Qcal.device)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_SELECT, Lq, Ksum.shape[2], device=Qcal.device)
    hils.hils_select(p, Qcal, Ksum, Bsum, idx, score, nsel, qpos=qpos, workspace=ws)
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "a bounded wait expired"
    return idx, score, nsel


def gpu_prefill(w, Q, K, V, idx, score, nsel, Kk=None, W=None):
    p = P(w, K=w.K if Kk is None else Kk, W=w.W if W is None else W)
    O = torch.full_like(Q, 99.0)
    lse = torch.full(Q.shape[:3], 99.0, dtype=torch.float32, device=Q.device)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_ATTEND_PREFILL, Q.shape[2], 0, device=Q.device)
    hils.hils_attend_prefill(p, Q, K, V, idx, score, nsel, O, lse, workspace=ws)
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "a bounded wait expired"
    return O, lse


def gpu_decode(w, Q, Kc, Vc, cache_len, idx, score, nsel, ws=None):
    p = P(w)
    if ws is None:
        ws = hils.alloc_workspace(p, hils.HILS_CALL_ATTEND_DECODE, 1, 0, device=Q.device)
    O = torch.full_like(Q, 99.0)
    lse = torch.full(Q.shape[:2], 99.0, dtype=torch.float32, device=Q.device)
    hils.hils_attend_decode(p, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse, workspace=ws)
    return O, lse


def to_dev(inp, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


PREFILL_CASES = {
    "cfg1_tiny_fp32": WORKLOADS[1],
    "cfg2_reduced_bf16": WORKLOADS[2].replace(H=4, N=1536 + 37),
    "bf16_d64": WORKLOADS[2].replace(H=3, d=64, N=700, K=5, W=100),
    "fp32_d128": WORKLOADS[1].replace(H=2, d=128, N=640 + 9, K=3, W=70),
}


# ------------------------------------------------------------------ summarise

@pytest.mark.parametrize("case", list(PREFILL_CASES))
def test_summarize_matches_oracle(oracle, cuda_device, case):
    w = PREFILL_CASES[case]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    ks_ref, bs_ref = oracle.summarize(inp["K"], inp["LQ"], 64, w.scale)
    assert_close(Ksum, ks_ref, w.dtype, "Ksum")
    assert np.abs(host(Bsum).double().numpy() - bs_ref).max() <= BSUM_ATOL


def test_summarize_full_prefill_workload(oracle, cuda_device):
    w = WORKLOADS[2]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    ks_ref, bs_ref = oracle.summarize(inp["K"], inp["LQ"], 64, w.scale)
    assert_close(Ksum, ks_ref, w.dtype, "Ksum")
    assert np.abs(host(Bsum).double().numpy() - bs_ref).max() <= BSUM_ATOL


def test_summarize_strided_views(oracle, cuda_device):
    """Keys inside a wider buffer, heads/batch permuted: strides are honoured."""
    w = WORKLOADS[2].replace(B=2, H=3, N=64 * 6)
    g = torch.Generator().manual_seed(5)
    big = torch.randn(3, 2, w.N, 2 * w.d, generator=g).to(w.dtype)
    K = big.permute(1, 0, 2, 3)[..., : w.d]          # [B,H,N,d], st = 2d, sb/sh swapped
    LQ = torch.randn(w.B, w.H, 6, w.d, generator=g).to(w.dtype)
    Kd = big.to(cuda_device).permute(1, 0, 2, 3)[..., : w.d]
    Ksum_buf = torch.zeros(w.B, w.H, 6, w.d + 8, dtype=w.dtype, device=cuda_device)
    Ksum = Ksum_buf[..., : w.d]
    Bsum = torch.empty(w.B, w.H, 6, dtype=torch.float32, device=cuda_device)
    hils.hils_summarize(P(w), Kd, LQ.to(cuda_device), Ksum, Bsum)
    ks_ref, bs_ref = oracle.summarize(K, LQ, 64, w.scale)
    assert_close(Ksum, ks_ref, w.dtype, "Ksum")
    assert (host(Ksum_buf[..., w.d:]) == 0).all(), "wrote outside the view"
    assert np.abs(host(Bsum).double().numpy() - bs_ref).max() <= BSUM_ATOL


# ------------------------------------------------------------------ select

@pytest.mark.parametrize("case", list(PREFILL_CASES) + ["cfg2_full"])
def test_select_prefill_bit_exact(oracle, cuda_device, case):
    w = WORKLOADS[2] if case == "cfg2_full" else PREFILL_CASES[case]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    i_ref, s_ref, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, w.K, w.scale)
    assert_same_selection(idx, nsel, i_ref, n_ref, case)
    scores_close(score, s_ref, n_ref, case)


def _decode_like(w, C, seed=3):
    B, H = w.B, w.H
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, H, 1, w.d, generator=g).to(w.dtype)
    Ksum = (torch.randn(B, H, C, w.d, generator=g) * 0.3).to(w.dtype)
    Bsum = (torch.rand(B, H, C, generator=g) * 4.0).float()
    return Q, Ksum, Bsum


@pytest.mark.parametrize("C,K,tpos", [(700, 16, None), (3000, 16, None), (20000, 32, None),
                                      (3000, 16, [1000, 64 * 3000 + 5])])
def test_select_split_paths_bit_exact(oracle, cuda_device, C, K, tpos):
    """Few queries, long contexts: the multi-CTA split search and its final merge."""
    w = WORKLOADS[4].replace(B=2, H=3, K=K)
    Q, Ksum, Bsum = _decode_like(w, C)
    B = Q.shape[0]
    qpos = torch.tensor([[64 * C + 3]] * B if tpos is None else [[t] for t in tpos], dtype=torch.int32)
    idx, score, nsel = gpu_select(w, Q.to(cuda_device), Ksum.to(cuda_device), Bsum.to(cuda_device),
                                  qpos=qpos.to(cuda_device))
    i_ref, s_ref, n_ref = oracle.select(Q, Ksum, Bsum, 64, K, w.scale, qpos=qpos)
    assert_same_selection(idx, nsel, i_ref, n_ref)
    scores_close(score, s_ref, n_ref)


@pytest.mark.parametrize("Hk", [0, 2])
def test_select_split_repeated_calls_on_one_workspace(oracle, cuda_device, Hk):
    """The decode select (screen, then the dependent-launched pick) called back to back
    on one workspace, cycling over three tables with nothing synchronising the calls:
    every call keeps the oracle's chunks bit-exactly (no call reads another's screen
    values), and the status word stays zero."""
    w = WORKLOADS[4].replace(B=1, H=8, K=16, Hk=Hk)
    C, G = 8191, w.H // w.Hkv
    qpos = torch.tensor([[64 * C + 3]], dtype=torch.int32)
    sets = []
    for seed in (11, 12, 13):
        Q, Ksum, Bsum = _decode_like(w, C, seed=seed)
        i_ref, _, n_ref = oracle.select(Q, Ksum, Bsum, 64, w.K, w.scale, qpos=qpos, group=G)
        sets.append((Q.to(cuda_device), Ksum.to(cuda_device), Bsum.to(cuda_device), i_ref, n_ref))
    p = P(w)
    qpos_d = qpos.to(cuda_device)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_SELECT, 1, C, device=cuda_device)
    outs = []
    for r in range(24):
        Q, Ksum, Bsum, _, _ = sets[r % 3]
        idx = torch.full((1, w.Hkv, 1, w.K), 7777, dtype=torch.int32, device=cuda_device)
        score = torch.full((1, w.H, 1, w.K), 7777.0, device=cuda_device)
        nsel = torch.full((1, w.Hkv, 1), 7777, dtype=torch.int32, device=cuda_device)
        hils.hils_select(p, Q, Ksum, Bsum, idx, score, nsel, qpos=qpos_d, workspace=ws)
        outs.append((idx, nsel))
    torch.cuda.synchronize()
    for r, (idx, nsel) in enumerate(outs):
        _, _, _, i_ref, n_ref = sets[r % 3]
        assert_same_selection(idx, nsel, i_ref, n_ref, f"call {r}")
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "a bounded wait expired"


def test_select_planted_exact_ties(oracle, cuda_device):
    """Twenty duplicated summaries give bit-identical scores above all others; only 16
    fit, and the lower chunk indices win. A second planted group ties lower down."""
    w = WORKLOADS[4].replace(B=2, H=3, K=16)
    C = 2500
    Q, Ksum, Bsum = _decode_like(w, C, seed=11)
    g = torch.Generator().manual_seed(12)
    dups = sorted(torch.randperm(C, generator=g)[:20].tolist())
    k0, b0 = Ksum[:, :, dups[0]].clone(), Bsum[:, :, dups[0]].clone() + 50.0
    for c in dups:
        Ksum[:, :, c] = k0
        Bsum[:, :, c] = b0
    qpos = torch.full((Q.shape[0], 1), 64 * C, dtype=torch.int32)
    idx, score, nsel = gpu_select(w, Q.to(cuda_device), Ksum.to(cuda_device), Bsum.to(cuda_device),
                                  qpos=qpos.to(cuda_device))
    assert (host(idx) == torch.tensor(dups[:16], dtype=torch.int32)).all()
    i_ref, s_ref, n_ref = oracle.select(Q, Ksum, Bsum, 64, w.K, w.scale, qpos=qpos)
    assert_same_selection(idx, nsel, i_ref, n_ref)
    # ties straddling the boundary: 10 clear winners, then 12 equal rows for 6 places
    Q, Ksum, Bsum = _decode_like(w, C, seed=13)
    rows = sorted(torch.randperm(C, generator=g)[:22].tolist())
    for c in rows[:10]:
        Bsum[:, :, c] += 80.0
    k0, b0 = Ksum[:, :, rows[10]].clone(), Bsum[:, :, rows[10]].clone() + 40.0
    for c in rows[10:]:
        Ksum[:, :, c] = k0
        Bsum[:, :, c] = b0
    idx, score, nsel = gpu_select(w, Q.to(cuda_device), Ksum.to(cuda_device), Bsum.to(cuda_device),
                                  qpos=qpos.to(cuda_device))
    want = torch.tensor(sorted(rows[:10] + rows[10:16]), dtype=torch.int32)
    assert (host(idx) == want).all()
    i_ref, s_ref, n_ref = oracle.select(Q, Ksum, Bsum, 64, w.K, w.scale, qpos=qpos)
    assert_same_selection(idx, nsel, i_ref, n_ref)


@pytest.mark.parametrize("C", [100, 5000])
def test_select_all_scores_equal(oracle, cuda_device, C):
    """Degenerate ranking (every chunk ties): the K lowest indices are kept."""
    w = WORKLOADS[4].replace(B=2, H=2, K=16)
    Q = torch.ones(2, 2, 1, w.d).to(w.dtype)
    Ksum = torch.ones(2, 2, C, w.d).to(w.dtype)
    Bsum = torch.full((2, 2, C), 0.5)
    qpos = torch.full((2, 1), 64 * C, dtype=torch.int32)
    idx, score, nsel = gpu_select(w, Q.to(cuda_device), Ksum.to(cuda_device), Bsum.to(cuda_device),
                                  qpos=qpos.to(cuda_device))
    assert (host(idx) == torch.arange(16, dtype=torch.int32)).all()
    i_ref, _, n_ref = oracle.select(Q, Ksum, Bsum, 64, w.K, w.scale, qpos=qpos)
    assert_same_selection(idx, nsel, i_ref, n_ref)


@pytest.mark.parametrize("K", [0, 1, 32])
def test_select_k_extremes(oracle, cuda_device, K):
    w = PREFILL_CASES["cfg2_reduced_bf16"]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum, K=K)
    i_ref, s_ref, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, K, w.scale)
    assert_same_selection(idx, nsel, i_ref, n_ref)
    if K:
        scores_close(score, s_ref, n_ref)


# many bf16 queries with d = 128 take the tensor-core select (scores in TMEM, one thread
# per query); these cases reach its column blocks, explicit positions, strided views and
# the exact fallback for rows with heavy ties

def _prefill_select_case(oracle, dev, w, qpos=None, Qcal=None, Ksum=None, Bsum=None, K=None):
    inp = make_prefill(w)
    d = to_dev(inp, dev)
    if Ksum is None:
        Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    Q = d["Qcal"] if Qcal is None else Qcal
    idx, score, nsel = gpu_select(w, Q, Ksum, Bsum, qpos=None if qpos is None else qpos.to(dev), K=K)
    i_ref, s_ref, n_ref = oracle.select(host(Q), host(Ksum), host(Bsum), 64, w.K if K is None else K, w.scale,
                                        qpos=qpos)
    assert_same_selection(idx, nsel, i_ref, n_ref)
    scores_close(score, s_ref, n_ref)
    return idx, nsel


@pytest.mark.parametrize("N", [64 * 300 + 17, 64 * 512 + 1, 64 * 513 + 5])
def test_select_tc_long_prefill(oracle, cuda_device, N):
    """300 chunks (column blocks of 256 + 64), the 512-column maximum, and 513 chunks
    (beyond TMEM: the warp kernel)."""
    w = WORKLOADS[2].replace(H=2 if N < 64 * 400 else 1, N=N)
    _prefill_select_case(oracle, cuda_device, w)


def test_select_tc_explicit_positions(oracle, cuda_device):
    """A later slice of a sequence: queries at t = 4096 + i against 96 chunks, plus a few
    rows moved before the first chunk and past the last."""
    w = WORKLOADS[2].replace(B=2, H=3, N=2048)
    inp = make_prefill(w)
    C = 96
    g = torch.Generator().manual_seed(21)
    Ksum = (torch.randn(w.B, w.H, C, w.d, generator=g) * 0.3).to(w.dtype)
    Bsum = torch.rand(w.B, w.H, C, generator=g) * 0.2 + 4.0
    qpos = (torch.arange(w.N, dtype=torch.int32) + 4096).repeat(w.B, 1)
    qpos[0, :5] = torch.tensor([0, 63, 64, 65, -3], dtype=torch.int32)
    qpos[1, -3:] = 64 * 200
    dev = cuda_device
    _prefill_select_case(oracle, dev, w, qpos=qpos, Qcal=inp["Qcal"].to(dev), Ksum=Ksum.to(dev),
                         Bsum=Bsum.to(dev))


def test_select_tc_strided_views(oracle, cuda_device):
    """Q~ and k' inside wider buffers with permuted batch and head strides."""
    w = WORKLOADS[2].replace(B=2, H=3, N=1000)
    C = w.N // 64
    g = torch.Generator().manual_seed(22)
    qbig = (torch.randn(w.H, w.B, w.N, 2 * w.d, generator=g) / 11.3).to(w.dtype).to(cuda_device)
    kbig = (torch.randn(w.H, w.B, C, w.d + 64, generator=g) * 0.3).to(w.dtype).to(cuda_device)
    Qcal = qbig.permute(1, 0, 2, 3)[..., w.d:]
    Ksum = kbig.permute(1, 0, 2, 3)[..., 64:]
    Bsum = (torch.rand(w.B, w.H, C, generator=g) * 0.3 + 4.0).to(cuda_device)
    _prefill_select_case(oracle, cuda_device, w, Qcal=Qcal, Ksum=Ksum, Bsum=Bsum)


@pytest.mark.parametrize("K", [1, 8, 28])
def test_select_tc_ties_fall_back_exactly(oracle, cuda_device, K):
    """Head 0: every summary equal (all rows tie). Head 1: twelve equal summaries on top
    (more band entries than the per-row capacity). Head 2: ordinary scores."""
    w = WORKLOADS[2].replace(H=3, N=64 * 60 + 9)
    C = w.N // 64
    g = torch.Generator().manual_seed(23)
    Ksum = (torch.randn(1, 3, C, w.d, generator=g) * 0.3).to(w.dtype)
    Bsum = torch.rand(1, 3, C, generator=g) * 0.2 + 4.0
    Ksum[0, 0] = Ksum[0, 0, 0].clone()
    Bsum[0, 0] = 4.1
    rows = torch.randperm(C, generator=g)[:12]
    Ksum[0, 1, rows] = Ksum[0, 1, rows[0]].clone()
    Bsum[0, 1, rows] = 9.0
    idx, nsel = _prefill_select_case(oracle, cuda_device, w, Qcal=make_prefill(w)["Qcal"].to(cuda_device),
                                     Ksum=Ksum.to(cuda_device), Bsum=Bsum.to(cuda_device), K=K)
    last = host(idx)[0, 0, -1]
    assert (last[:K] == torch.arange(K, dtype=torch.int32)).all()  # ties: lowest indices


def test_select_without_chunks(cuda_device):
    """Sequences shorter than one chunk: nothing is eligible."""
    w = WORKLOADS[2].replace(H=2, N=40)
    inp = to_dev(make_prefill(w), cuda_device)
    Ksum = torch.empty(1, 2, 0, w.d, dtype=w.dtype, device=cuda_device)
    Bsum = torch.empty(1, 2, 0, device=cuda_device)
    idx, score, nsel = gpu_select(w, inp["Qcal"], Ksum, Bsum)
    assert (host(nsel) == 0).all() and (host(idx) == -1).all()


# ------------------------------------------------------------------ attend

@pytest.mark.parametrize("case", list(PREFILL_CASES))
def test_attend_prefill_matches_oracle(oracle, cuda_device, case):
    w = PREFILL_CASES[case]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                   64, w.W, w.scale)
    assert_close(O, O_ref, w.dtype, "O")
    assert_close(lse, lse_ref, torch.float32, "lse")


@pytest.mark.parametrize("Kk,W", [(0, 64), (4, 0), (0, 0), (4, 5000)])
def test_attend_prefill_degenerate_terms(oracle, cuda_device, Kk, W):
    """Window only, chunks only, nothing (o = 0, lse = -inf), window longer than the sequence."""
    w = WORKLOADS[2].replace(H=2, N=300, K=Kk, W=W)
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                   64, W, w.scale)
    assert_close(O, O_ref, w.dtype, "O")
    assert_close(lse, lse_ref, torch.float32, "lse")


def test_attend_prefill_exact_mass_is_block_sparse_attention(oracle, cuda_device):
    """Scores replaced by exact log Z_{i,c}, every eligible chunk kept, W = 0: the kernel
    computes plain softmax attention over the complete chunks before the query."""
    w = WORKLOADS[2].replace(H=2, N=64 * 9, K=8, W=0)
    inp = make_prefill(w)
    N = w.N
    idx = np.full((1, 2, N, 8), -1, np.int32)
    nsel = np.zeros((1, 2, N), np.int32)
    for i in range(N):
        ne = min(i // 64, 8)
        idx[:, :, i, :ne] = np.arange(ne)
        nsel[:, :, i] = ne
    score = oracle.chunk_logmass(inp["Q"], inp["K"], idx, nsel, 64, w.scale).astype(np.float32)
    d = to_dev(inp, cuda_device)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], torch.from_numpy(idx).to(cuda_device),
                         torch.from_numpy(score).to(cuda_device), torch.from_numpy(nsel).to(cuda_device))
    Qd, Kd, Vd = (inp[k][0].double() for k in ("Q", "K", "V"))
    ref = np.zeros((2, N, w.d))
    for h in range(2):
        for i in range(64, N):
            ne = i // 64
            lg = (Kd[h, : ne * 64] @ Qd[h, i]) * w.scale
            ref[h, i] = (torch.softmax(lg, 0) @ Vd[h, : ne * 64]).numpy()
    assert_close(O[0, :, 64:], ref[:, 64:], w.dtype, "O")


@pytest.mark.parametrize("B,H,N,K,W", [(2, 8, 4096 + 100, 16, 512), (1, 6, 64 * 50 + 200, 3, 100),
                                         (2, 3, 64 * 130 + 63, 32, 300)])
def test_attend_prefill_persistent_items(oracle, cuda_device, B, H, N, K, W):
    """More 256-query work items than SMs (each persistent CTA runs several, with
    ragged last items and both query tiles partly past N), B > 1, K = 3 (few shared
    chunks: many tiles with one empty half) and K = 32."""
    w = WORKLOADS[2].replace(B=B, H=H, N=N, K=K, W=W)
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                   64, w.W, w.scale)
    assert_close(O, O_ref, w.dtype, "O")
    assert_close(lse, lse_ref, torch.float32, "lse")


def test_attend_prefill_full_size(oracle, cuda_device):
    """The 8K prefill workload (B=1, H=32, N=8192, K=16, W=512) in the launch
    configuration the benchmark times: every output of every head against the oracle
    (fed the GPU's selection), per head and over the whole tensor."""
    w = WORKLOADS[2]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel), 64, w.W,
                                   w.scale)
    for h in range(w.H):
        sl = slice(h, h + 1)
        assert_close(O[:, sl], O_ref[:, sl], w.dtype, f"O head {h}")
        assert_close(lse[:, sl], lse_ref[:, sl], torch.float32, f"lse head {h}")
    assert_close(O, O_ref, w.dtype, "O")


def test_prefill_query_locality_workload(oracle, cuda_device):
    """The 8K prefill with slowly changing Q_cal (adjacent queries keep overlapping chunk
    sets), four heads: selection bit-exact, outputs within tolerance, and each
    256-query item's union of kept chunks far below the eligible count, which is the
    regime of the query-packing kernel."""
    w = WORKLOADS[6].replace(H=4)
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    i_ref, s_ref, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, w.K, w.scale)
    assert_same_selection(idx, nsel, i_ref, n_ref, "local")
    scores_close(score, s_ref, n_ref, "local")
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                   64, w.W, w.scale)
    assert_close(O, O_ref, w.dtype, "O")
    assert_close(lse, lse_ref, torch.float32, "lse")
    ih = host(idx).reshape(w.B, w.H, w.N // 256, 256 * w.K).numpy()
    unions = [len(set(r.tolist()) - {-1}) for r in ih.reshape(-1, 256 * w.K)[w.H:]]  # items past the first
    assert np.mean(unions) < 40, np.mean(unions)


def test_bounded_waits_expire_and_recover(oracle, cuda_device):
    """The tensor-core select and prefill attend with every wait on work in progress made
    to expire at its first check (HILS_FLAG_DIAG_EXPIRE_WAITS): each call returns with
    bit 0 of its status word set and every output left as it was (the copies and
    tensor-core operations started before the expiry are drained, tensor memory is
    released); then the same calls with the normal time limit give the oracle's
    results."""
    w = WORKLOADS[2].replace(H=2, N=1536 + 37)  # 3146 queries: the tensor-core select
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    pd = P(w, flags=hils.HILS_FLAG_DIAG_EXPIRE_WAITS)
    B, H, N, K = w.B, w.H, w.N, w.K
    # select
    ws = hils.alloc_workspace(pd, hils.HILS_CALL_SELECT, N, Ksum.shape[2], device=cuda_device)
    idx = torch.full((B, H, N, K), 7777, dtype=torch.int32, device=cuda_device)
    score = torch.full((B, H, N, K), 7777.0, device=cuda_device)
    nsel = torch.full((B, H, N), 7777, dtype=torch.int32, device=cuda_device)
    hils.hils_select(pd, d["Qcal"], Ksum, Bsum, idx, score, nsel, workspace=ws)
    torch.cuda.synchronize()
    assert int(host(ws[:4]).view(torch.int32)[0]) & 1, "select: no wait expired"
    i1, s1, n1 = gpu_select(w, d["Qcal"], Ksum, Bsum)
    i_ref, _, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, K, w.scale)
    assert_same_selection(i1, n1, i_ref, n_ref, "select after the diagnostic call")
    assert (host(nsel) == 7777).all() and (host(idx) == 7777).all() and (host(score) == 7777.0).all(), \
        "the diagnostic select wrote outputs"
    # prefill attend
    wsa = hils.alloc_workspace(pd, hils.HILS_CALL_ATTEND_PREFILL, N, 0, device=cuda_device)
    O = torch.full_like(d["Q"], 99.0)
    lse = torch.full((B, H, N), 99.0, device=cuda_device)
    hils.hils_attend_prefill(pd, d["Q"], d["K"], d["V"], i1, s1, n1, O, lse, workspace=wsa)
    torch.cuda.synchronize()
    assert int(host(wsa[:4]).view(torch.int32)[0]) & 1, "attend: no wait expired"
    O1, l1 = gpu_prefill(w, d["Q"], d["K"], d["V"], i1, s1, n1)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(i1), host(s1), host(n1), 64, w.W, w.scale)
    assert_close(O1, O_ref, w.dtype, "O after the diagnostic call")
    assert_close(l1, lse_ref, torch.float32, "lse after the diagnostic call")
    assert (host(lse) == 99.0).all() and (host(O).float() == 99.0).all(), "the diagnostic attend wrote outputs"


def _decode_small(cuda_device, lens=(5000, 3001), K=16, W=512, H=3):
    w = WORKLOADS[4].replace(B=len(lens), H=H, N=max(lens), K=K, W=W, needles=0)
    inp = make_decode(w)
    inp["cache_len"] = torch.tensor(lens, dtype=torch.int32)
    return w, inp


def test_attend_decode_matches_oracle(oracle, cuda_device):
    w, inp = _decode_small(cuda_device)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    qpos = (inp["cache_len"] - 1).reshape(w.B, 1)
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum, qpos=qpos.to(cuda_device))
    i_ref, s_ref, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, w.K, w.scale, qpos=qpos)
    assert_same_selection(idx, nsel, i_ref, n_ref)
    ws = hils.alloc_workspace(P(w), hils.HILS_CALL_ATTEND_DECODE, 1, 0, device=cuda_device)
    for rep in range(2):  # the second call checks that the arrival counters were reset
        O, lse = gpu_decode(w, d["Q"], d["K"], d["V"], d["cache_len"], idx, score, nsel, ws=ws)
        O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                       64, w.W, w.scale, qpos=qpos)
        assert_close(O, O_ref, w.dtype, f"O rep {rep}")
        assert_close(lse, lse_ref[:, :, 0], torch.float32, f"lse rep {rep}")


@pytest.mark.parametrize("lens,K,W", [((1, 63, 64, 65), 4, 512), ((129, 700), 32, 1024),
                                      ((2000, 1500), 0, 100), ((2000, 1500), 8, 0)])
def test_attend_decode_edges(oracle, cuda_device, lens, K, W):
    """Tiny caches (first token, one chunk), K = 32, window-only and chunk-only decode."""
    w, inp = _decode_small(cuda_device, lens=lens, K=K, W=W, H=2)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    qpos = (inp["cache_len"] - 1).reshape(w.B, 1)
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum, qpos=qpos.to(cuda_device))
    O, lse = gpu_decode(w, d["Q"], d["K"], d["V"], d["cache_len"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                   64, W, w.scale, qpos=qpos)
    assert_close(O, O_ref, w.dtype, "O")
    assert_close(lse, lse_ref[:, :, 0], torch.float32, "lse")


# ------------------------------------------------------------------ chained

@pytest.mark.parametrize("case", ["cfg1_tiny_fp32", "cfg2_reduced_bf16"])
def test_end_to_end_against_chained_oracle(oracle, cuda_device, case):
    """GPU summarise -> select -> attend against the oracle's own chain, whose summary
    table is stored in the input dtype like the GPU's. Selections may differ only where
    the oracle's K-th and (K+1)-th scores lie within 1e-6; outputs are compared on
    every query whose selection agrees."""
    w = PREFILL_CASES[case]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, _ = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)

    ks, bs = oracle.summarize(inp["K"], inp["LQ"], 64, w.scale)
    ks_t = torch.from_numpy(ks).to(w.dtype)
    bs_t = torch.from_numpy(bs).float()
    i_ref, s_ref, n_ref = oracle.select(inp["Qcal"], ks_t, bs_t, 64, w.K, w.scale)
    allsc = oracle.score_all(inp["Qcal"], ks_t, bs_t, 64, w.scale)
    O_ref, _ = oracle.attend(inp["Q"], inp["K"], inp["V"], i_ref, s_ref, n_ref, 64, w.W, w.scale)
    ig = host(idx).numpy()
    differ = (ig != i_ref).any(-1)
    for b, h, i in np.argwhere(differ):
        srt = np.sort(allsc[b, h, i][np.isfinite(allsc[b, h, i])])[::-1]
        assert len(srt) > w.K and srt[w.K - 1] - srt[w.K] <= 1e-6, "selection differs outside a near-tie"
    same = ~differ
    assert same.mean() > 0.98
    Og = host(O).double().numpy()
    assert_close(torch.from_numpy(Og[same]), O_ref[same], w.dtype, "O")


# ------------------------------------------------------------------ full sizes

def _decode_chain(w, d, Ksum, Bsum, ws=None):
    p = P(w)
    B, H, Hk = w.B, w.H, w.Hkv
    idx = torch.full((B, Hk, 1, w.K), 7777, dtype=torch.int32, device=Ksum.device)
    score = torch.full((B, H, 1, w.K), 7777.0, device=Ksum.device)
    nsel = torch.full((B, Hk, 1), 7777, dtype=torch.int32, device=Ksum.device)
    O = torch.full_like(d["Q"], 99.0)
    lse = torch.full((B, H), 99.0, device=Ksum.device)
    if ws is None:
        ws = hils.alloc_workspace(p, hils.HILS_CALL_DECODE, 1, Ksum.shape[2], device=Ksum.device)
    hils.hils_decode(p, d["Qcal"], Ksum, Bsum, d["Q"], d["K"], d["V"], d["cache_len"], idx, score, nsel, O, lse,
                     workspace=ws)
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "a bounded wait expired"
    return idx, score, nsel, O, lse, ws


@pytest.mark.parametrize("case", ["small16", "small6", "full"])
def test_decode_chain_equals_separate_calls(oracle, cuda_device, case):
    """hils_decode (the select and the attend as one chain, the attend's window tiles
    not waiting for the select) keeps exactly the chunks and scores of hils_select and
    gives the outputs of hils_attend_decode within the output tolerance; the small case
    is also checked against the oracle, and every case runs twice on one workspace."""
    full = case == "full"
    if full:
        w = WORKLOADS[4]
        d = make_decode(w, device=cuda_device)
    else:
        w, inp = _decode_small(cuda_device, lens=(12001, 9000), H=8 if case == "small16" else 3)
        d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    qpos = (d["cache_len"] - 1).reshape(w.B, 1).contiguous()
    i1, s1, n1 = gpu_select(w, d["Qcal"], Ksum, Bsum, qpos=qpos)
    O1, l1 = gpu_decode(w, d["Q"], d["K"], d["V"], d["cache_len"], i1, s1, n1)
    ws = None
    for rep in range(2):
        i2, s2, n2, O2, l2, ws = _decode_chain(w, d, Ksum, Bsum, ws)
        assert torch.equal(i1, i2) and torch.equal(n1, n2) and torch.equal(s1, s2), f"selection rep {rep}"
        assert_close(O2, host(O1).double().numpy(), w.dtype, f"O rep {rep}")
        assert np.abs(host(l2).double().numpy() - host(l1).double().numpy()).max() <= 1e-4, f"lse rep {rep}"
    if not full:
        i_ref, _, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, w.K, w.scale, qpos=host(qpos))
        assert_same_selection(i2, n2, i_ref, n_ref)
        O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(i2), host(s2), host(n2), 64, w.W,
                                       w.scale, qpos=host(qpos))
        assert_close(O2, O_ref, w.dtype, "O")
        assert_close(l2, lse_ref[:, :, 0], torch.float32, "lse")
    del d
    torch.cuda.empty_cache()


@pytest.mark.parametrize("lens,K,W,d,dtype", [
    ((1, 65, 700, 12001), 16, 512, 128, torch.bfloat16),   # no chunk, all kept, short table, long
    ((3000, 70000, 9000, 64 * 1000), 32, 1024, 128, torch.bfloat16),
    ((5000, 12345, 64, 8000), 8, 0, 128, torch.bfloat16),  # no window
    ((4000, 9001, 20000, 130), 16, 300, 64, torch.bfloat16),
    ((3000, 9001, 700, 6000), 16, 512, 128, torch.float32),
])
def test_decode_chain_edges(oracle, cuda_device, lens, K, W, d, dtype):
    """hils_decode with B*H = 16 queries against the oracle and the separate calls:
    empty tables, tables of at most K chunks, fewer than K+1 groups, no window, K = 32,
    d = 64 and float32."""
    w = WORKLOADS[4].replace(B=len(lens), H=4, N=max(lens), K=K, W=W, d=d, dtype=dtype, needles=0)
    inp = make_decode(w)
    inp["cache_len"] = torch.tensor(lens, dtype=torch.int32)
    dv = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, dv["K"], dv["LQ"])
    qpos = (dv["cache_len"] - 1).reshape(w.B, 1).contiguous()
    i1, s1, n1 = gpu_select(w, dv["Qcal"], Ksum, Bsum, qpos=qpos)
    O1, l1 = gpu_decode(w, dv["Q"], dv["K"], dv["V"], dv["cache_len"], i1, s1, n1)
    i2, s2, n2, O2, l2, _ = _decode_chain(w, dv, Ksum, Bsum)
    assert torch.equal(i1, i2) and torch.equal(n1, n2) and torch.equal(s1, s2)
    i_ref, s_ref, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, K, w.scale, qpos=host(qpos))
    assert_same_selection(i2, n2, i_ref, n_ref)
    scores_close(s2, s_ref, n_ref, "hils_decode scores")
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(i2), host(s2), host(n2), 64, W, w.scale,
                                   qpos=host(qpos))
    assert_close(O2, O_ref, dtype, "O")
    fin = np.isfinite(lse_ref[:, :, 0])
    l2h = host(l2).double().numpy()
    assert (np.isfinite(l2h) == fin).all()
    assert np.abs(l2h[fin] - lse_ref[:, :, 0][fin]).max() <= 1e-4
    assert_close(O2, host(O1).double().numpy(), dtype, "O vs separate calls")


@pytest.mark.parametrize("cfg", [3, 4, 5, 9])
def test_decode_workload_full_size(oracle, cuda_device, cfg):
    """Decode workloads at full size, generated on the GPU: summaries sampled, the
    selection of every (b, h) bit-exact, outputs of sampled (b, h) within tolerance."""
    w = WORKLOADS[cfg]
    inp = make_decode(w, device=cuda_device)
    Ksum, Bsum = gpu_summarize(w, inp["K"], inp["LQ"])
    qpos = (inp["cache_len"] - 1).reshape(w.B, 1)
    idx, score, nsel = gpu_select(w, inp["Qcal"], Ksum, Bsum, qpos=qpos)
    i_ref, s_ref, n_ref = oracle.select(host(inp["Qcal"]), host(Ksum), host(Bsum), 64, w.K, w.scale,
                                        qpos=host(qpos))
    assert_same_selection(idx, nsel, i_ref, n_ref, f"cfg{cfg}")
    scores_close(score, s_ref, n_ref, f"cfg{cfg}")
    if w.needle_landmark:  # retrieval: every needle's chunk is kept
        ih, nh = host(idx).numpy(), host(nsel).numpy()
        for b in range(w.B):
            for h in range(w.Hkv):
                kept = set(ih[b, h, 0, : nh[b, h, 0]].tolist())
                assert set((inp["needles"][b, h] // 64).tolist()) <= kept, (b, h)
    O, lse = gpu_decode(w, inp["Q"], inp["K"], inp["V"], inp["cache_len"], idx, score, nsel)
    # the whole step in one call (the launch configuration the benchmark times): the same
    # selection, and the outputs of the separate calls within rounding
    i2, s2, n2, O2, l2, _ = _decode_chain(w, inp, Ksum, Bsum)
    assert torch.equal(idx, i2) and torch.equal(nsel, n2) and torch.equal(score, s2), f"cfg{cfg} hils_decode"
    assert_close(O2, host(O).double().numpy(), w.dtype, "O hils_decode vs separate calls")
    assert np.abs(host(l2).double().numpy() - host(lse).double().numpy()).max() <= 1e-4
    g = torch.Generator().manual_seed(cfg)
    for _ in range(3):
        b = int(torch.randint(0, w.B, (1,), generator=g))
        h = int(torch.randint(0, w.H, (1,), generator=g))
        Kh = host(inp["K"][b:b + 1, h:h + 1])
        Vh = host(inp["V"][b:b + 1, h:h + 1])
        LQh = host(inp["LQ"][b:b + 1, h:h + 1])
        c0 = 137  # summaries of a run of chunks of this head
        ks_ref, bs_ref = oracle.summarize(Kh[:, :, : 64 * (c0 + 40)], LQh[:, :, : c0 + 40], 64, w.scale)
        assert_close(Ksum[b:b + 1, h:h + 1, c0:c0 + 40], ks_ref[:, :, c0:], w.dtype, "Ksum")
        assert np.abs(host(Bsum[b:b + 1, h:h + 1, c0:c0 + 40]).double().numpy() - bs_ref[:, :, c0:]).max() \
            <= BSUM_ATOL
        O_ref, lse_ref = oracle.attend(host(inp["Q"][b:b + 1, h:h + 1]), Kh, Vh,
                                       host(idx[b:b + 1, h:h + 1]), host(score[b:b + 1, h:h + 1]),
                                       host(nsel[b:b + 1, h:h + 1]), 64, w.W, w.scale,
                                       qpos=host(qpos[b:b + 1]))
        assert_close(O[b:b + 1, h:h + 1], O_ref, w.dtype, f"O b{b} h{h}")
        assert_close(O2[b:b + 1, h:h + 1], O_ref, w.dtype, f"O hils_decode b{b} h{h}")
        assert abs(float(lse[b, h]) - lse_ref[0, 0, 0]) <= 1e-4
        assert abs(float(l2[b, h]) - lse_ref[0, 0, 0]) <= 1e-4
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("d", [128, 64])
def test_screen_radius_covers_the_float64_score(oracle, cuda_device, d):
    """The decode-shaped select writes every eligible chunk's float32 screen value s_c and
    radius e_c to its workspace (B*H*Lq*C float pairs after the 256-byte status header,
    which must stay zero). The kept set is only exact if |s_c - x_c| <= e_c, with x_c the
    oracle's float64 score: check it for every chunk; check that the radius is the
    fused-multiply-add bound scale |q| |k'| (d+2) 2^-23 + |s| 2^-22 (within its own float32
    rounding), and that the observed error stays well inside it (1/4), so the bound is
    not merely lucky."""
    w = WORKLOADS[4].replace(B=2, H=4, d=d, K=16)
    C = 5000
    g = torch.Generator().manual_seed(31)
    Q = torch.randn(w.B, w.H, 1, d, generator=g).to(w.dtype)
    Ksum = (torch.randn(w.B, w.H, C, d, generator=g) * torch.rand(w.B, w.H, C, 1, generator=g) * 2).to(w.dtype)
    Bsum = (torch.rand(w.B, w.H, C, generator=g) * 4.0).float()
    qpos = torch.full((w.B, 1), 64 * C + 10, dtype=torch.int32)
    p = P(w)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_SELECT, 1, C, device=cuda_device)
    assert ws is not None
    idx = torch.empty(w.B, w.H, 1, w.K, dtype=torch.int32, device=cuda_device)
    score = torch.empty(w.B, w.H, 1, w.K, device=cuda_device)
    nsel = torch.empty(w.B, w.H, 1, dtype=torch.int32, device=cuda_device)
    hils.hils_select(p, Q.to(cuda_device), Ksum.to(cuda_device), Bsum.to(cuda_device), idx, score, nsel,
                     qpos=qpos.to(cuda_device), workspace=ws)
    torch.cuda.synchronize()
    wsh = host(ws)
    assert (wsh[:256] == 0).all()
    scr = wsh[256:].view(torch.float32)[: w.B * w.H * C * 2].reshape(w.B, w.H, C, 2).double().numpy()
    x = oracle.score_all(Q, Ksum, Bsum, 64, w.scale, qpos=qpos)[:, :, 0, :]
    err = np.abs(scr[..., 0] - x)
    assert (err <= scr[..., 1]).all(), f"radius violated: {float((err - scr[..., 1]).max()):.3e}"
    qn = np.linalg.norm(Q.double().numpy(), axis=-1)            # [B,H,1]
    kn = np.linalg.norm(Ksum.double().numpy(), axis=-1)         # [B,H,C]
    fma = w.scale * qn * kn * (d + 2) * 2.0 ** -23 + np.abs(x) * 2.0 ** -22
    assert np.allclose(scr[..., 1], fma, rtol=1e-5, atol=0), "radius is not the fused-multiply-add bound"
    assert (err / scr[..., 1]).max() <= 1 / 4, f"observed error {float((err / scr[..., 1]).max()):.3f} of the bound"
    i_ref, s_ref, n_ref = oracle.select(Q, Ksum, Bsum, 64, w.K, w.scale, qpos=qpos)
    assert_same_selection(idx, nsel, i_ref, n_ref)


@pytest.mark.parametrize("cfg,Hk,dtype,d", [(4, 0, torch.bfloat16, 128), (8, 2, torch.bfloat16, 128),
                                             (4, 0, torch.float32, 64)])
def test_summarize_append_decode_time(oracle, cuda_device, cfg, Hk, dtype, d):
    """hils_summarize_append summarises exactly the chunk each sequence's newest token
    completed (cache_len a positive multiple of 64), with the bits of the full pass, and
    leaves every other entry of the table untouched."""
    w = WORKLOADS[cfg].replace(B=5, H=4, Hk=Hk, d=d, dtype=dtype, N=64 * 40, needles=0)
    inp = make_decode(w)
    dv = to_dev(inp, cuda_device)
    Ksum_full, Bsum_full = gpu_summarize(w, dv["K"], dv["LQ"])
    lens = [64 * 17, 64 * 17 + 5, 64, 1, 64 * 40]
    cache_len = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    Ksum = torch.full_like(Ksum_full, 7.0)
    Bsum = torch.full_like(Bsum_full, 99.0)
    hils.hils_summarize_append(P(w), dv["K"], cache_len, dv["LQ"], Ksum, Bsum)
    torch.cuda.synchronize()
    done = {b: L // 64 - 1 for b, L in enumerate(lens) if L >= 64 and L % 64 == 0}
    assert done == {0: 16, 2: 0, 4: 39}
    for b in range(w.B):
        for c in range(w.C):
            if done.get(b) == c:
                assert torch.equal(Ksum[b, :, c], Ksum_full[b, :, c]), (b, c)
                assert torch.equal(Bsum[b, :, c], Bsum_full[b, :, c]), (b, c)
            else:
                assert (Ksum[b, :, c] == 7.0).all() and (Bsum[b, :, c] == 99.0).all(), (b, c)
    # the appended chunk of sequence 0 against the oracle
    ks_ref, bs_ref = oracle.summarize(inp["K"][:1, :, : 64 * 17], inp["LQ"][:1, :, :17], 64, w.scale)
    assert_close(Ksum[:1, :, 16], ks_ref[:, :, 16], dtype, "Ksum")
    assert np.abs(host(Bsum[:1, :, 16]).double().numpy() - bs_ref[:, :, 16]).max() <= BSUM_ATOL
