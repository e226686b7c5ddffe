"""The FMA-pipe helpers of the tensor-core prefill attend, checked directly: 2^x by a
fitted polynomial and 1/z by an integer seed and two Newton steps, evaluated on the GPU
through hils_selftest_fast_math and compared with float64 references over their whole
input ranges (x in [-125, 127]; normal positive z across the exponent range), at the
relative error bounds their header states: 2.4e-7 and 7e-6."""
import numpy as np
import pytest
import torch

import hierarchical_chunk_sparse_b200 as hils

pytestmark = pytest.mark.gpu


def _run(x, z, dev):
    xd, zd = torch.from_numpy(x).to(dev), torch.from_numpy(z).to(dev)
    e, r = torch.empty_like(xd), torch.empty_like(zd)
    hils.hils_selftest_fast_math(xd, zd, e, r)
    torch.cuda.synchronize()
    return e.cpu().numpy().astype(np.float64), r.cpu().numpy().astype(np.float64)


def test_exp2_and_reciprocal_within_their_bounds(cuda_device):
    rng = np.random.default_rng(20260709)
    n = 1 << 24
    # x: a dense grid over [-125, 127] plus random points and the integers (f = 0)
    x = np.concatenate([np.linspace(-125.0, 127.0, n // 2), rng.uniform(-125.0, 127.0, n // 2 - 253),
                        np.arange(-125, 128)]).astype(np.float32)
    # z: log-uniform over normal floats 2^-125 .. 2^125, plus a dense grid of one binade
    z = np.concatenate([np.exp2(rng.uniform(-125.0, 125.0, n // 2)),
                        np.linspace(1.0, 2.0, n // 2)]).astype(np.float32)
    e, r = _run(x, z, cuda_device)
    e_ref = np.exp2(x.astype(np.float64))
    r_ref = 1.0 / z.astype(np.float64)
    e_rel = np.abs(e - e_ref) / e_ref
    r_rel = np.abs(r - r_ref) / r_ref
    print(f"exp2 max rel {e_rel.max():.3e} at x={x[e_rel.argmax()]}; recip max rel {r_rel.max():.3e} "
          f"at z={z[r_rel.argmax()]}")
    assert e_rel.max() <= 2.4e-7
    assert r_rel.max() <= 7e-6


def test_exp2_clamps_below_the_normal_range(cuda_device):
    """Arguments below -125 give the value at -125, a normal float within the bound of
    2^-125."""
    x = np.array([-126.0, -150.0, -1e30, -125.0], np.float32)
    e, _ = _run(x, np.ones_like(x), cuda_device)
    assert (e == e[-1]).all()
    assert abs(e[-1] - 2.0 ** -125) <= 2.4e-7 * 2.0 ** -125
