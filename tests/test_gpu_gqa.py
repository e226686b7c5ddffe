"""GPU parity of grouped-query attention ("Hierarchical Sparse Attention Done Right",
summary page, Methodology 3, GQA adaptation): G query heads share a key-value head and
keep the chunks with the largest maximum of their chunk scores, each head weighting them
with its own score. Every stage against the float64 oracle's grouped routines, with the
bars of the multi-head parity tests: selections bit-exact, scores within
1e-5 + 2e-6 |s|, bf16 outputs max-abs 2e-2 and relative L2 1e-2, float32 1e-4."""
import numpy as np
import pytest
import torch

from hils_synth import WORKLOADS, make_decode, make_prefill
from hils_testutil import BSUM_ATOL, assert_close, assert_same_selection, host, scores_close
from test_gpu_parity import _decode_chain, gpu_decode, gpu_prefill, gpu_select, gpu_summarize, to_dev

pytestmark = pytest.mark.gpu

PREFILL_GQA = {
    "bf16_d128_g4": WORKLOADS[7].replace(H=8, N=1536 + 37),
    "bf16_d128_g8_b2": WORKLOADS[7].replace(B=2, H=8, Hk=1, N=64 * 20 + 5, K=5, W=200),
    "bf16_d64_g2": WORKLOADS[7].replace(H=6, Hk=3, d=64, N=700, K=5, W=100),
    "fp32_d128_g2": WORKLOADS[1].replace(H=4, Hk=2, d=128, N=640 + 9, K=3, W=70),
    "fp32_d64_g3": WORKLOADS[1].replace(H=3, Hk=1, N=512 + 33, K=4, W=64),
    # tensor-core select: three heads per group (one operand buffer reloaded), and two
    # heads with 256 TMEM columns each
    "bf16_d128_g3_tc": WORKLOADS[7].replace(H=6, Hk=2, N=1536 + 37),
    "bf16_d128_g2_tc_long": WORKLOADS[7].replace(H=4, Hk=2, N=64 * 200 + 5, K=8, W=256),
    # three heads whose tables exceed the TMEM columns: the warp-per-query group kernel
    "bf16_d128_g3_warp_long": WORKLOADS[7].replace(H=3, Hk=1, N=64 * 180 + 7, K=8, W=256),
}


def _per_head(nsel, G):
    return np.repeat(np.asarray(nsel), G, axis=1)


def _select_and_check(oracle, w, inp, d, qpos=None):
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum, qpos=None if qpos is None else qpos.to(d["K"].device))
    i_ref, s_ref, n_ref = oracle.select(host(d["Qcal"]), host(Ksum), host(Bsum), 64, w.K, w.scale,
                                        qpos=qpos, group=w.G)
    assert_same_selection(idx, nsel, i_ref, n_ref, "group selection")
    scores_close(score, s_ref, _per_head(n_ref, w.G), "per-head scores")
    return Ksum, Bsum, idx, score, nsel


@pytest.mark.parametrize("case", list(PREFILL_GQA))
def test_gqa_summarize(oracle, cuda_device, case):
    """Each query head's landmark query attends over its key-value head's chunk."""
    w = PREFILL_GQA[case]
    inp = make_prefill(w)
    assert inp["K"].shape[1] == w.Hkv and inp["LQ"].shape[1] == w.H
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    ks_ref, bs_ref = oracle.summarize(inp["K"], inp["LQ"], 64, w.scale)
    assert_close(Ksum, ks_ref, w.dtype, "Ksum")
    assert np.abs(host(Bsum).double().numpy() - bs_ref).max() <= BSUM_ATOL


@pytest.mark.parametrize("case", list(PREFILL_GQA))
def test_gqa_prefill_select_and_attend(oracle, cuda_device, case):
    """Group selection bit-exact and per-head scores; then the attend (tensor-core path
    for bf16 d = 128, the general path otherwise) against the oracle fed the GPU's own
    selection."""
    w = PREFILL_GQA[case]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    _, _, idx, score, nsel = _select_and_check(oracle, w, inp, d)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                   64, w.W, w.scale)
    assert_close(O, O_ref, w.dtype, "O")
    assert_close(lse, lse_ref, torch.float32, "lse")


def test_gqa_prefill_persistent_items(oracle, cuda_device):
    """More 256-query items than SMs with B = 2 and groups of 4: every persistent CTA
    runs several items of different key-value heads."""
    w = WORKLOADS[7].replace(B=2, H=16, Hk=4, N=4096 + 100)
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    _, _, idx, score, nsel = _select_and_check(oracle, w, inp, d)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                   64, w.W, w.scale)
    assert_close(O, O_ref, w.dtype, "O")
    assert_close(lse, lse_ref, torch.float32, "lse")


def test_gqa_prefill_full_size(oracle, cuda_device):
    """The grouped 8K prefill (32 query heads, 8 key-value heads) in the launch
    configuration the benchmark times: every selection bit-exact, the outputs of two
    sampled groups (all their heads) against the oracle."""
    w = WORKLOADS[7]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    _, _, idx, score, nsel = _select_and_check(oracle, w, inp, d)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    g = torch.Generator().manual_seed(77)
    for hk in torch.randperm(w.Hkv, generator=g)[:2].tolist():
        sq, sk = slice(hk * w.G, (hk + 1) * w.G), slice(hk, hk + 1)
        O_ref, lse_ref = oracle.attend(inp["Q"][:, sq], inp["K"][:, sk], inp["V"][:, sk], host(idx[:, sk]),
                                       host(score[:, sq]), host(nsel[:, sk]), 64, w.W, w.scale)
        assert_close(O[:, sq], O_ref, w.dtype, f"O group {hk}")
        assert_close(lse[:, sq], lse_ref, torch.float32, f"lse group {hk}")


@pytest.mark.parametrize("lens,H,Hk,K,W,d,dtype", [
    ((12001, 9000), 8, 2, 16, 512, 128, torch.bfloat16),
    ((1, 65, 700, 5000), 4, 1, 32, 1024, 128, torch.bfloat16),
    ((3000, 2000), 6, 3, 8, 0, 128, torch.bfloat16),    # groups of 3: a CTA per head
    ((2000, 1500), 8, 4, 0, 100, 128, torch.bfloat16),
    ((3000, 7001), 8, 1, 16, 300, 64, torch.bfloat16),  # groups of 8, d = 64
    ((4000, 2500), 4, 2, 8, 200, 128, torch.float32),
])
def test_gqa_decode(oracle, cuda_device, lens, H, Hk, K, W, d, dtype):
    """Decode with ragged cache lengths (first token, one chunk, fewer chunks than K),
    no window, window only, groups of 2, 3, 4 and 8, d = 64 and float32: the separate
    select and attend, then hils_decode as one chain on the same inputs, all against
    the oracle."""
    w = WORKLOADS[8].replace(B=len(lens), H=H, Hk=Hk, N=max(lens), K=K, W=W, d=d, dtype=dtype, needles=0)
    inp = make_decode(w)
    inp["cache_len"] = torch.tensor(lens, dtype=torch.int32)
    d = to_dev(inp, cuda_device)
    qpos = (inp["cache_len"] - 1).reshape(w.B, 1)
    Ksum, Bsum, idx, score, nsel = _select_and_check(oracle, w, inp, d, qpos=qpos)
    O, lse = gpu_decode(w, d["Q"], d["K"], d["V"], d["cache_len"], idx, score, nsel)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel),
                                   64, W, w.scale, qpos=qpos)
    assert_close(O, O_ref, w.dtype, "O")
    fin = np.isfinite(lse_ref[:, :, 0])
    lh = host(lse).double().numpy()
    assert (np.isfinite(lh) == fin).all()
    if fin.any():
        assert np.abs(lh[fin] - lse_ref[:, :, 0][fin]).max() <= 1e-4
    if K > 0:
        i2, s2, n2, O2, l2, _ = _decode_chain(w, d, Ksum, Bsum)
        assert torch.equal(idx, i2) and torch.equal(nsel, n2) and torch.equal(score, s2)
        assert_close(O2, O_ref, w.dtype, "O (hils_decode)")


def test_gqa_decode_full_size(oracle, cuda_device):
    """The grouped 512K decode (32 query heads, 8 key-value heads, one needle per
    key-value head), generated on the GPU: every group's selection bit-exact, outputs
    of two sampled groups within tolerance, hils_decode equal to the separate calls."""
    w = WORKLOADS[8]
    inp = make_decode(w, device=cuda_device)
    qpos = (inp["cache_len"] - 1).reshape(w.B, 1)
    Ksum, Bsum, idx, score, nsel = _select_and_check(oracle, w, inp, inp, qpos=host(qpos))
    O, lse = gpu_decode(w, inp["Q"], inp["K"], inp["V"], inp["cache_len"], idx, score, nsel)
    g = torch.Generator().manual_seed(88)
    for hk in torch.randperm(w.Hkv, generator=g)[:2].tolist():
        sq, sk = slice(hk * w.G, (hk + 1) * w.G), slice(hk, hk + 1)
        O_ref, lse_ref = oracle.attend(host(inp["Q"][:, sq]), host(inp["K"][:, sk]), host(inp["V"][:, sk]),
                                       host(idx[:, sk]), host(score[:, sq]), host(nsel[:, sk]), 64, w.W, w.scale,
                                       qpos=host(qpos))
        assert_close(O[:, sq], O_ref, w.dtype, f"O group {hk}")
        assert np.abs(host(lse[:, sq]).double().numpy() - lse_ref[:, :, 0]).max() <= 1e-4
    i2, s2, n2, O2, l2, _ = _decode_chain(w, inp, Ksum, Bsum)
    assert torch.equal(idx, i2) and torch.equal(nsel, n2) and torch.equal(score, s2)
    assert_close(O2, host(O).double().numpy(), w.dtype, "O (hils_decode)")
    del inp
    torch.cuda.empty_cache()
