"""GPU parity of the backward pass (fixed selection) against the float64 autograd oracle
(``oracle/backward.py``, pinned by finite differences): the GPU's forward chain
(summarise, select, attend) gives the selection, O and lse; the three backward calls
then give dscore, dQ, dK, dV, dQcal, dKsum, dBsum and dLQ, each compared with the
oracle's gradient of sum(O * dO) for the same selection. Bars, as relative L2 error of
each gradient: float32 inputs 1e-5 (float32 arithmetic and atomic accumulation order;
observed about 5e-7); bf16 inputs 1e-2, the forward's bar (the forward's O and summary
table are stored in bf16, which moves D_i and the chunk scores by up to 2^-9 relative,
and the tensor-core products take dO, dl and cv rounded to bf16; observed about 3e-3).
Element-wise, every gradient's largest error is within twice that bar times the
gradient's largest magnitude. The cases cover K = 0 (no kept chunk), W = 0 (no window),
a table of 400 chunks (chunk 0's list of thousands of queries is cut into runs of 1024),
grouped heads and a window longer than a run. The last test makes every bounded wait
of the tensor-core walk expire."""
import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_b200 as hils
from hils_synth import WORKLOADS, make_prefill
from hils_testutil import host
from oracle import backward as ob
from test_gpu_parity import P, gpu_prefill, gpu_select, gpu_summarize, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    "fp32_d64": (WORKLOADS[1].replace(H=2, N=64 * 5 + 17, K=3, W=70), 1e-5),
    "fp32_d128_grouped": (WORKLOADS[1].replace(H=4, Hk=2, d=128, N=64 * 4 + 9, K=2, W=90), 1e-5),
    "bf16_d128": (WORKLOADS[2].replace(H=2, N=64 * 6 + 9, K=4, W=100), 1e-2),
    "bf16_d64_grouped": (WORKLOADS[7].replace(H=4, Hk=1, d=64, N=64 * 5 + 3, K=3, W=130), 1e-2),
    # no kept chunk (K = 0): the window alone carries every gradient; dscore is empty
    "bf16_d128_K0": (WORKLOADS[2].replace(H=2, N=64 * 6 + 9, K=0, W=100), 1e-2),
    "fp32_d64_K0": (WORKLOADS[1].replace(H=2, N=64 * 5 + 17, K=0, W=70), 1e-5),
    # no window (W = 0): the kept chunks alone
    "bf16_d128_W0": (WORKLOADS[2].replace(H=2, N=64 * 6 + 9, K=4, W=0), 1e-2),
    "fp32_d128_W0_grouped": (WORKLOADS[1].replace(H=4, Hk=2, d=128, N=64 * 4 + 9, K=2, W=0), 1e-5),
    # 400 chunks: chunk 0's list of thousands of queries is cut into several runs of the
    # tensor-core walk, and the score backward sorts and sums a large table (its k' copy
    # still fits in shared memory)
    "bf16_d128_C400": (WORKLOADS[2].replace(H=1, N=64 * 400, K=16, W=512), 1e-2),
    # the tensor-core walk (bf16, d = 128) with query heads sharing a kept list
    "bf16_d128_grouped": (WORKLOADS[7].replace(H=4, Hk=2, d=128, N=64 * 5 + 3, K=3, W=130), 1e-2),
    # fewer tokens than one chunk (C = 0): no summary, nothing kept; dQcal is zero
    "bf16_d128_N40": (WORKLOADS[2].replace(H=2, N=40, K=4, W=16), 1e-2),
    # a window longer than one work item's 1024 queries: each window block's queries are
    # cut into two runs, whose dK and dV shares add up
    "bf16_d128_W1500": (WORKLOADS[2].replace(H=1, N=64 * 40 + 5, K=4, W=1500), 1e-2),
}


def _max_abs(g, r):
    """Largest element-wise error, relative to the largest reference magnitude."""
    g = host(g).double().numpy() if isinstance(g, torch.Tensor) else np.asarray(g, np.float64)
    r = r.numpy() if isinstance(r, torch.Tensor) else np.asarray(r, np.float64)
    if r.size == 0:
        return 0.0
    top = float(np.abs(r).max())
    err = float(np.abs(g - r).max())
    return err / top if top > 0 else err


def _rel(g, r):
    g = host(g).double().numpy() if isinstance(g, torch.Tensor) else np.asarray(g, np.float64)
    r = r.numpy() if isinstance(r, torch.Tensor) else np.asarray(r, np.float64)
    if r.size == 0:
        return 0.0
    den = np.linalg.norm(r)
    return float(np.linalg.norm(g - r) / den) if den > 0 else float(np.abs(g).max())


@pytest.mark.parametrize("case", list(CASES))
def test_backward_matches_oracle(cuda_device, case):
    w, tol = CASES[case]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    g = torch.Generator().manual_seed(7)
    dO = torch.randn(O.shape, generator=g).to(cuda_device)
    p = P(w)
    B, H, N, dd, Hk, K, C = w.B, w.H, w.N, w.d, w.Hkv, w.K, w.C
    f32 = dict(dtype=torch.float32, device=cuda_device)
    dQ, dK, dV = torch.empty(B, H, N, dd, **f32), torch.zeros(B, Hk, N, dd, **f32), torch.zeros(B, Hk, N, dd, **f32)
    dscore = torch.empty(B, H, N, K, **f32)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_ATTEND_BACKWARD, N, 0, device=cuda_device)
    hils.hils_attend_prefill_backward(p, d["Q"], d["K"], d["V"], idx, score, nsel, O, lse, dO, dQ, dK, dV, dscore,
                                      workspace=ws)
    dQcal = torch.empty(B, H, N, dd, **f32)
    dKsum, dBsum = torch.zeros(B, H, C, dd, **f32), torch.zeros(B, H, C, **f32)
    hils.hils_select_backward(p, d["Qcal"], Ksum, idx, nsel, dscore, dQcal, dKsum, dBsum)
    dLQ = torch.empty(B, H, C, dd, **f32)
    hils.hils_summarize_backward(p, d["K"], d["LQ"], dKsum, dBsum, dK, dLQ)
    torch.cuda.synchronize()
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "a bounded wait of the attend backward expired"
    ref = ob.grads(inp["Q"], inp["K"], inp["V"], inp["Qcal"], inp["LQ"], host(idx), host(nsel), host(dO), 64, w.W,
                   w.scale, batch=256)
    errs = {
        "dscore": _rel(dscore, ref["dscore"]),
        "dQ": _rel(dQ, ref["dQ"]),
        "dV": _rel(dV, ref["dV"]),
        "dQcal": _rel(dQcal, ref["dQcal"]),
        "dKsum": _rel(dKsum, ref["dKsum"]),
        "dBsum": _rel(dBsum, ref["dBsum"]),
        "dLQ": _rel(dLQ, ref["dLQ"]),
        "dK": _rel(dK, ref["dK"]),
    }
    maxe = {k: _max_abs(g_, ref[k]) for k, g_ in (("dscore", dscore), ("dQ", dQ), ("dV", dV), ("dQcal", dQcal),
                                                    ("dKsum", dKsum), ("dBsum", dBsum), ("dLQ", dLQ), ("dK", dK))}
    print(case, {k: f"{v:.2e}" for k, v in errs.items()}, "max-abs", {k: f"{v:.2e}" for k, v in maxe.items()})
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"relative L2 errors above {tol}: {bad} (all: {errs})"
    bad = {k: v for k, v in maxe.items() if not v <= 2 * tol}
    assert not bad, f"max-abs errors above {2 * tol} of the largest gradient: {bad} (all: {maxe})"
    # padding of dscore is exactly zero
    kept = torch.arange(K, device=cuda_device).view(1, 1, 1, K) < nsel.repeat_interleave(w.G, dim=1).unsqueeze(-1)
    assert (dscore[~kept] == 0).all()


FULL = {
    # the 8K prefill (B1 H32 d128 N8192, K16, W512): two sampled query heads
    "prefill8k": (2, 2),
    # the grouped 8K prefill (32 query heads, 8 key-value heads): one sampled group
    "prefill8k_grouped": (7, 1),
}


@pytest.mark.parametrize("case", list(FULL))
def test_backward_full_size(cuda_device, case):
    """The 8K prefill backward at full size, in the launch configuration the benchmark
    times (forward chain, then the three backward calls with an allocated workspace):
    for sampled key-value heads, every gradient of that head's slice (dscore, dQ, dQcal
    of its query heads; dK, dV; dKsum, dBsum, dLQ) against the float64 oracle, which
    runs over blocks of 256 query rows and sums the blocks' gradients. Heads and groups
    are independent, so a slice's gradients are its own problem's. Bar as above for
    bf16 inputs."""
    wid, nsample = FULL[case]
    w = WORKLOADS[wid]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    g = torch.Generator().manual_seed(17)
    dO = torch.randn(O.shape, generator=g).to(cuda_device)
    p = P(w)
    B, H, N, dd, Hk, K, C, G = w.B, w.H, w.N, w.d, w.Hkv, w.K, w.C, w.G
    f32 = dict(dtype=torch.float32, device=cuda_device)
    dQ, dK, dV = torch.empty(B, H, N, dd, **f32), torch.zeros(B, Hk, N, dd, **f32), torch.zeros(B, Hk, N, dd, **f32)
    dscore, dQcal = torch.empty(B, H, N, K, **f32), torch.empty(B, H, N, dd, **f32)
    dKsum, dBsum, dLQ = torch.zeros(B, H, C, dd, **f32), torch.zeros(B, H, C, **f32), torch.empty(B, H, C, dd, **f32)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_ATTEND_BACKWARD, N, 0, device=cuda_device)
    hils.hils_attend_prefill_backward(p, d["Q"], d["K"], d["V"], idx, score, nsel, O, lse, dO, dQ, dK, dV, dscore,
                                      workspace=ws)
    hils.hils_select_backward(p, d["Qcal"], Ksum, idx, nsel, dscore, dQcal, dKsum, dBsum)
    hils.hils_summarize_backward(p, d["K"], d["LQ"], dKsum, dBsum, dK, dLQ)
    torch.cuda.synchronize()
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "a bounded wait of the attend backward expired"
    kept = torch.arange(K, device=cuda_device).view(1, 1, 1, K) < nsel.repeat_interleave(G, dim=1).unsqueeze(-1)
    assert (dscore[~kept] == 0).all()
    dO_h = host(dO)
    for hk in torch.randperm(Hk, generator=g)[:nsample].tolist():
        qs, ks = slice(hk * G, (hk + 1) * G), slice(hk, hk + 1)
        ref = ob.grads(inp["Q"][:, qs], inp["K"][:, ks], inp["V"][:, ks], inp["Qcal"][:, qs], inp["LQ"][:, qs],
                       host(idx[:, ks]), host(nsel[:, ks]), dO_h[:, qs], 64, w.W, w.scale, batch=256)
        errs = {
            "dscore": _rel(dscore[:, qs], ref["dscore"]),
            "dQ": _rel(dQ[:, qs], ref["dQ"]),
            "dQcal": _rel(dQcal[:, qs], ref["dQcal"]),
            "dK": _rel(dK[:, ks], ref["dK"]),
            "dV": _rel(dV[:, ks], ref["dV"]),
            "dKsum": _rel(dKsum[:, qs], ref["dKsum"]),
            "dBsum": _rel(dBsum[:, qs], ref["dBsum"]),
            "dLQ": _rel(dLQ[:, qs], ref["dLQ"]),
        }
        maxe = {
            "dscore": _max_abs(dscore[:, qs], ref["dscore"]),
            "dQ": _max_abs(dQ[:, qs], ref["dQ"]),
            "dQcal": _max_abs(dQcal[:, qs], ref["dQcal"]),
            "dK": _max_abs(dK[:, ks], ref["dK"]),
            "dV": _max_abs(dV[:, ks], ref["dV"]),
            "dKsum": _max_abs(dKsum[:, qs], ref["dKsum"]),
            "dBsum": _max_abs(dBsum[:, qs], ref["dBsum"]),
            "dLQ": _max_abs(dLQ[:, qs], ref["dLQ"]),
        }
        print(case, hk, {k: f"{v:.2e}" for k, v in errs.items()}, "max-abs", {k: f"{v:.2e}" for k, v in maxe.items()})
        bad = {k: v for k, v in errs.items() if not v <= 1e-2}
        assert not bad, f"kv head {hk}: relative L2 errors above 1e-2: {bad} (all: {errs})"
        bad = {k: v for k, v in maxe.items() if not v <= 2e-2}
        assert not bad, f"kv head {hk}: max-abs errors above 2e-2 of the largest gradient: {bad} (all: {maxe})"


def test_backward_waits_expire_and_recover(cuda_device):
    """The tensor-core attend backward (bf16, d = 128) with every wait on work in progress
    made to expire at its first check (HILS_FLAG_DIAG_EXPIRE_WAITS): the call returns
    with bit 0 of its status word set, dK and dV (accumulated) left as they were, dQ and
    dscore as the call's own clearing left them (zero); then the same call with the normal
    time limit gives the oracle's gradients."""
    w = WORKLOADS[2].replace(H=2, N=64 * 6 + 9, K=4, W=100)
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    g = torch.Generator().manual_seed(7)
    dO = torch.randn(O.shape, generator=g).to(cuda_device)
    B, H, N, dd, Hk, K = w.B, w.H, w.N, w.d, w.Hkv, w.K
    f32 = dict(dtype=torch.float32, device=cuda_device)
    dQ, dscore = torch.full((B, H, N, dd), 5.0, **f32), torch.full((B, H, N, K), 5.0, **f32)
    dK, dV = torch.full((B, Hk, N, dd), 3.0, **f32), torch.full((B, Hk, N, dd), 3.0, **f32)
    pd = P(w, flags=hils.HILS_FLAG_DIAG_EXPIRE_WAITS)
    ws = hils.alloc_workspace(pd, hils.HILS_CALL_ATTEND_BACKWARD, N, 0, device=cuda_device)
    hils.hils_attend_prefill_backward(pd, d["Q"], d["K"], d["V"], idx, score, nsel, O, lse, dO, dQ, dK, dV, dscore,
                                      workspace=ws)
    torch.cuda.synchronize()
    assert int(host(ws[:4]).view(torch.int32)[0]) & 1, "no wait expired"
    assert (host(dK) == 3.0).all() and (host(dV) == 3.0).all(), "the diagnostic call added to dK or dV"
    assert (host(dQ) == 0.0).all() and (host(dscore) == 0.0).all(), "the diagnostic call wrote dQ or dscore"
    p = P(w)
    dK.zero_()
    dV.zero_()
    hils.hils_attend_prefill_backward(p, d["Q"], d["K"], d["V"], idx, score, nsel, O, lse, dO, dQ, dK, dV, dscore,
                                      workspace=ws)
    torch.cuda.synchronize()
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "the status word was not cleared by the normal call"
    full = ob.grads(inp["Q"], inp["K"], inp["V"], inp["Qcal"], inp["LQ"], host(idx), host(nsel), host(dO), 64, w.W,
                    w.scale, batch=256)
    # the attend call's own gradients (dK also takes the summaries' share, added later)
    for name, got in (("dQ", dQ), ("dV", dV), ("dscore", dscore)):
        assert _rel(got, full[name]) <= 1e-2, f"{name} after the diagnostic call"


def test_backward_unaligned_gradients(cuda_device):
    """Gradient arrays need only 4-byte alignment: with dQ, dK, dV, dKsum and dBsum
    starting 4 bytes past a 16-byte boundary the kernels take their scalar-atomic forms
    (the vector adds need 16-byte rows); the gradients match the oracle as before."""
    w = WORKLOADS[2].replace(H=2, N=64 * 6 + 9, K=4, W=100)
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = gpu_select(w, d["Qcal"], Ksum, Bsum)
    O, lse = gpu_prefill(w, d["Q"], d["K"], d["V"], idx, score, nsel)
    g = torch.Generator().manual_seed(7)
    dO = torch.randn(O.shape, generator=g).to(cuda_device)
    p = P(w)
    B, H, N, dd, Hk, K, C = w.B, w.H, w.N, w.d, w.Hkv, w.K, w.C

    def offset(*shape):  # a dense float32 tensor whose data starts 4 bytes past 16-byte alignment
        n = 1
        for s in shape:
            n *= s
        base = torch.zeros(n + 4, dtype=torch.float32, device=cuda_device)
        t = base[1:n + 1].view(*shape)
        assert t.data_ptr() % 16 == 4
        return t

    dQ, dK, dV = offset(B, H, N, dd), offset(B, Hk, N, dd), offset(B, Hk, N, dd)
    dscore = torch.empty(B, H, N, K, dtype=torch.float32, device=cuda_device)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_ATTEND_BACKWARD, N, 0, device=cuda_device)
    hils.hils_attend_prefill_backward(p, d["Q"], d["K"], d["V"], idx, score, nsel, O, lse, dO, dQ, dK, dV, dscore,
                                      workspace=ws)
    dQcal = offset(B, H, N, dd)
    dKsum, dBsum = offset(B, H, C, dd), offset(B, H, C)
    hils.hils_select_backward(p, d["Qcal"], Ksum, idx, nsel, dscore, dQcal, dKsum, dBsum)
    dLQ = offset(B, H, C, dd)
    hils.hils_summarize_backward(p, d["K"], d["LQ"], dKsum, dBsum, dK, dLQ)
    torch.cuda.synchronize()
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0
    ref = ob.grads(inp["Q"], inp["K"], inp["V"], inp["Qcal"], inp["LQ"], host(idx), host(nsel), host(dO), 64, w.W,
                   w.scale, batch=256)
    for name, got in (("dQ", dQ), ("dK", dK), ("dV", dV), ("dscore", dscore), ("dQcal", dQcal), ("dKsum", dKsum),
                      ("dBsum", dBsum), ("dLQ", dLQ)):
        assert _rel(got, ref[name]) <= 1e-2, f"{name}: {_rel(got, ref[name])}"
