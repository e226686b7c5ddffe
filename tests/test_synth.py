"""The seeded input generators (no GPU): determinism and the planted structure."""
import torch

from hils_synth import WORKLOADS, make_prefill


def test_prefill_generator_is_deterministic():
    w = WORKLOADS[2].replace(H=2, N=640)
    a, b = make_prefill(w), make_prefill(w)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_query_locality_workload_structure():
    """Workload 6: Q_cal is one base vector per 256-token block plus 0.25 x iid noise, so
    neighbours inside a block point the same way and blocks are unrelated; the iid
    prefill workload has no such structure. Everything else keeps workload 2's recipe."""
    w6 = WORKLOADS[6].replace(H=2, N=1024)
    q = make_prefill(w6)["Qcal"].float()
    cos = torch.nn.functional.cosine_similarity
    inside = cos(q[..., 1:256, :], q[..., :255, :], dim=-1)
    assert float(inside.mean()) > 0.9 and float(inside.min()) > 0.6
    across = cos(q[..., 255::256, :][..., :3, :], q[..., 256::256, :], dim=-1)
    assert float(across.abs().max()) < 0.5
    # scale: each component is N(0, 1 + 0.25^2) / d before bf16 rounding
    var = float(q.var()) * w6.d
    assert abs(var - (1 + 0.25 ** 2)) < 0.1
    w2 = WORKLOADS[2].replace(H=2, N=1024)
    q2 = make_prefill(w2)["Qcal"].float()
    assert float(cos(q2[..., 1:, :], q2[..., :-1, :], dim=-1).abs().mean()) < 0.15
    assert (w6.B, w6.d, w6.K, w6.W, w6.S, w6.dtype) == (w2.B, w2.d, w2.K, w2.W, w2.S, w2.dtype)
