"""hils_attend_decode_noalloc: the decode attend for callers that cannot allocate
device memory (a plug-in handed only pointers and a stream, code under a fixed memory
budget). Its scratch is a fixed array inside the library instead of a caller-provided
workspace. This file is collected last, so a stop at its first failure has already
run every other test; it also passes on its own in a fresh process."""
import pytest
import torch

import hierarchical_chunk_sparse_b200 as hils
from hils_synth import WORKLOADS, make_decode
from hils_testutil import assert_close

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode(oracle, cuda_device):
    w = WORKLOADS[4].replace(B=2, H=4, N=6000, needles=0)
    inp = make_decode(w)
    inp["cache_len"] = torch.tensor([6000, 4097], dtype=torch.int32)
    d = {k: v.to(cuda_device) for k, v in inp.items() if isinstance(v, torch.Tensor)}
    p = hils.Params(B=w.B, H=w.H, d=w.d, K=w.K, W=w.W, dtype=w.dtype)
    C = w.N // 64
    Ksum = torch.empty(w.B, w.H, C, w.d, dtype=w.dtype, device=cuda_device)
    Bsum = torch.empty(w.B, w.H, C, dtype=torch.float32, device=cuda_device)
    hils.hils_summarize(p, d["K"], d["LQ"], Ksum, Bsum)
    qpos = (d["cache_len"] - 1).reshape(w.B, 1).contiguous()
    idx = torch.empty(w.B, w.H, 1, w.K, dtype=torch.int32, device=cuda_device)
    score = torch.empty(w.B, w.H, 1, w.K, dtype=torch.float32, device=cuda_device)
    nsel = torch.empty(w.B, w.H, 1, dtype=torch.int32, device=cuda_device)
    ws_sel = hils.alloc_workspace(p, hils.HILS_CALL_SELECT, 1, C, device=cuda_device)
    hils.hils_select(p, d["Qcal"], Ksum, Bsum, idx, score, nsel, qpos=qpos, workspace=ws_sel)

    ws = hils.alloc_workspace(p, hils.HILS_CALL_ATTEND_DECODE, 1, 0, device=cuda_device)
    O_ref = torch.empty_like(d["Q"])
    lse_ref = torch.empty(w.B, w.H, dtype=torch.float32, device=cuda_device)
    hils.hils_attend_decode(p, d["Q"], d["K"], d["V"], d["cache_len"], idx, score, nsel, O_ref, lse_ref,
                            workspace=ws)
    ref = O_ref.double().cpu().numpy()
    # the float64 oracle fed the same selection
    O_or, lse_or = oracle.attend(inp["Q"], inp["K"], inp["V"], idx.cpu(), score.cpu(), nsel.cpu(), 64, w.W,
                                 w.scale, qpos=qpos.cpu())
    for call in range(2):  # the second call reuses the scratch left by the first
        O = torch.full_like(d["Q"], 7.0)
        lse = torch.full((w.B, w.H), 7.0, dtype=torch.float32, device=cuda_device)
        hils.hils_attend_decode_noalloc(p, d["Q"], d["K"], d["V"], d["cache_len"], idx, score, nsel, O, lse)
        torch.cuda.synchronize()
        assert_close(O, ref, w.dtype, f"O call {call}")
        assert_close(lse, lse_ref.double().cpu().numpy(), torch.float32, f"lse call {call}")
        assert_close(O, O_or, w.dtype, f"O call {call} vs oracle")
        assert_close(lse, lse_or[:, :, 0], torch.float32, f"lse call {call} vs oracle")


def test_noalloc_rejects_bad_arguments_before_any_work(cuda_device):
    """A misaligned output view is rejected with the same status as hils_attend_decode,
    before the call queues anything."""
    p = hils.Params(B=1, H=2, d=128, K=4, W=64, dtype=torch.bfloat16)
    Q = torch.zeros(1, 2, 1, 128, dtype=torch.bfloat16, device=cuda_device)
    KV = torch.zeros(1, 2, 640, 128, dtype=torch.bfloat16, device=cuda_device)
    cl = torch.full((1,), 640, dtype=torch.int32, device=cuda_device)
    idx = torch.zeros(1, 2, 1, 4, dtype=torch.int32, device=cuda_device)
    sc = torch.zeros(1, 2, 1, 4, device=cuda_device)
    ns = torch.zeros(1, 2, 1, dtype=torch.int32, device=cuda_device)
    O = torch.zeros(1, 2, 1, 136, dtype=torch.bfloat16, device=cuda_device)[..., 1:129]  # 2-byte offset
    with pytest.raises(hils.HilsError) as err:
        hils.hils_attend_decode_noalloc(p, Q, KV, KV, cl, idx, sc, ns, O)
    assert err.value.status == 3


def test_noalloc_rejects_problems_beyond_its_capacity(cuda_device):
    """B=64, H=32, K=32, W=1024: about 25 MiB of scratch, more than the 4 MiB built in."""
    p = hils.Params(B=64, H=32, d=128, K=32, W=1024, dtype=torch.bfloat16)
    assert hils.hils_workspace_bytes(p, hils.HILS_CALL_ATTEND_DECODE, 1, 0) > 4 << 20
    Q = torch.zeros(64, 32, 1, 128, dtype=torch.bfloat16, device=cuda_device)
    KV = torch.zeros(64, 32, 64, 128, dtype=torch.bfloat16, device=cuda_device)
    cl = torch.full((64,), 64, dtype=torch.int32, device=cuda_device)
    idx = torch.zeros(64, 32, 1, 32, dtype=torch.int32, device=cuda_device)
    sc = torch.zeros(64, 32, 1, 32, device=cuda_device)
    ns = torch.zeros(64, 32, 1, dtype=torch.int32, device=cuda_device)
    with pytest.raises(hils.HilsError) as err:
        hils.hils_attend_decode_noalloc(p, Q, KV, KV, cl, idx, sc, ns, torch.empty_like(Q))
    assert err.value.status == 4
