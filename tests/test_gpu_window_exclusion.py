"""GPU parity of the window-exclusion variant (`HILS_FLAG_EXCLUDE_WINDOW_CHUNKS`: chunks
lying wholly inside the query's window are not selected) against the oracle's
`exclude_window`, on every select path: the tensor-core prefill select (one head and
grouped heads), the warp kernel (float32), the decode screen and pick (one head and
grouped heads) and the `hils_decode` chain. Selections bit-exact, outputs within the
parity tolerances."""
import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_b200 as hils
from hils_synth import WORKLOADS, make_decode, make_prefill
from hils_testutil import assert_close, assert_same_selection, host, scores_close
from test_gpu_parity import gpu_summarize, to_dev

pytestmark = pytest.mark.gpu
FLAG = hils.HILS_FLAG_EXCLUDE_WINDOW_CHUNKS


def _params(w, flags=FLAG):
    return hils.Params(B=w.B, H=w.H, d=w.d, K=w.K, W=w.W, dtype=w.dtype, H_kv=w.Hk, flags=flags)


def _select(w, Qcal, Ksum, Bsum, qpos=None):
    p = _params(w)
    B, H, Lq, Hk, k = Qcal.shape[0], Qcal.shape[1], Qcal.shape[2], w.Hkv, w.K
    dev = Qcal.device
    idx = torch.full((B, Hk, Lq, k), 7777, dtype=torch.int32, device=dev)
    score = torch.full((B, H, Lq, k), 7777.0, device=dev)
    nsel = torch.full((B, Hk, Lq), 7777, dtype=torch.int32, device=dev)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_SELECT, Lq, Ksum.shape[2], device=dev)
    hils.hils_select(p, Qcal, Ksum, Bsum, idx, score, nsel, qpos=qpos, workspace=ws)
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "a bounded wait expired"
    return idx, score, nsel


PREFILL = {
    "bf16_tc": WORKLOADS[2].replace(H=4, N=1536 + 37, W=300),
    "bf16_tc_aligned_window": WORKLOADS[2].replace(H=2, N=2048, W=256),
    "fp32_warp": WORKLOADS[1].replace(H=2, N=640 + 9, K=3, W=130),
    "bf16_tc_grouped": WORKLOADS[7].replace(H=8, N=1536 + 37, W=300),
}


@pytest.mark.parametrize("case", list(PREFILL))
def test_window_exclusion_prefill(oracle, cuda_device, case):
    w = PREFILL[case]
    inp = make_prefill(w)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    idx, score, nsel = _select(w, d["Qcal"], Ksum, Bsum)
    i_ref, s_ref, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, w.K, w.scale, group=w.G,
                                        exclude_window=w.W)
    assert_same_selection(idx, nsel, i_ref, n_ref, case)
    scores_close(score, s_ref, np.repeat(n_ref, w.G, axis=1), case)
    # no kept chunk lies wholly inside its query's window
    t = np.arange(w.N)[None, None, :, None]
    ih = host(idx).numpy()
    w0 = np.maximum(0, t - w.W + 1)
    assert ((ih < 0) | (ih * 64 < w0)).all()
    # the attend over the variant's selection
    p = _params(w)
    O = torch.empty_like(d["Q"])
    lse = torch.empty(d["Q"].shape[:3], dtype=torch.float32, device=cuda_device)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_ATTEND_PREFILL, w.N, 0, device=cuda_device)
    hils.hils_attend_prefill(p, d["Q"], d["K"], d["V"], idx, score, nsel, O, lse, workspace=ws)
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel), 64, w.W,
                                   w.scale)
    assert_close(O, O_ref, w.dtype, "O")
    assert_close(lse, lse_ref, torch.float32, "lse")


@pytest.mark.parametrize("lens,H,Hk,W", [((12001, 9000), 4, 0, 512), ((12001, 64 * 100), 4, 0, 3000),
                                         ((20000, 7777), 8, 2, 2048)])
def test_window_exclusion_decode_chain(oracle, cuda_device, lens, H, Hk, W):
    """hils_decode with the flag (screen and pick, one head or grouped heads), against
    the oracle's selection and attend."""
    w = WORKLOADS[8].replace(B=len(lens), H=H, Hk=Hk, N=max(lens), W=W, needles=0)
    inp = make_decode(w)
    inp["cache_len"] = torch.tensor(lens, dtype=torch.int32)
    d = to_dev(inp, cuda_device)
    Ksum, Bsum = gpu_summarize(w, d["K"], d["LQ"])
    p = _params(w)
    B, Hkv, k = w.B, w.Hkv, w.K
    idx = torch.full((B, Hkv, 1, k), 7777, dtype=torch.int32, device=cuda_device)
    score = torch.full((B, H, 1, k), 7777.0, device=cuda_device)
    nsel = torch.full((B, Hkv, 1), 7777, dtype=torch.int32, device=cuda_device)
    O = torch.empty_like(d["Q"])
    lse = torch.empty(B, H, device=cuda_device)
    ws = hils.alloc_workspace(p, hils.HILS_CALL_DECODE, 1, Ksum.shape[2], device=cuda_device)
    hils.hils_decode(p, d["Qcal"], Ksum, Bsum, d["Q"], d["K"], d["V"], d["cache_len"], idx, score, nsel, O, lse,
                     workspace=ws)
    assert int(host(ws[:4]).view(torch.int32)[0]) == 0, "a bounded wait expired"
    qpos = (inp["cache_len"] - 1).reshape(B, 1)
    i_ref, s_ref, n_ref = oracle.select(inp["Qcal"], host(Ksum), host(Bsum), 64, k, w.scale, qpos=qpos, group=w.G,
                                        exclude_window=W)
    assert_same_selection(idx, nsel, i_ref, n_ref, "decode")
    scores_close(score, s_ref, np.repeat(n_ref, w.G, axis=1), "decode")
    O_ref, lse_ref = oracle.attend(inp["Q"], inp["K"], inp["V"], host(idx), host(score), host(nsel), 64, W,
                                   w.scale, qpos=qpos)
    assert_close(O, O_ref, w.dtype, "O")
    assert np.abs(host(lse).double().numpy() - lse_ref[:, :, 0]).max() <= 1e-4
