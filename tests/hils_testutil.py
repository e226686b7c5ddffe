"""Helpers shared by the GPU parity tests: tolerances, CPU copies, chained runs."""
from __future__ import annotations

import numpy as np
import torch

# Output tolerances: bf16 results max-abs 2e-2 and relative L2 1e-2; float32 1e-4.
TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-4)}
BSUM_ATOL = 1e-4


def host(t: torch.Tensor) -> torch.Tensor:
    return t.detach().to("cpu")


def assert_close(gpu, ref, dtype, what=""):
    """Max-abs and relative-L2 check of a GPU result against a float64 oracle array."""
    g = host(gpu).double().numpy() if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    atol, rtol = TOL[dtype]
    fin = np.isfinite(r)
    assert (np.isfinite(g) == fin).all(), f"{what}: finite pattern differs"
    diff = np.abs(g[fin] - r[fin])
    max_abs = float(diff.max()) if diff.size else 0.0
    denom = float(np.linalg.norm(r[fin]))
    rel = float(np.linalg.norm(g[fin] - r[fin]) / denom) if denom > 0 else max_abs
    assert max_abs <= atol, f"{what}: max abs err {max_abs:.3e} > {atol} (worst row: {_worst_row(g, r)})"
    assert rel <= rtol, f"{what}: rel L2 err {rel:.3e} > {rtol} (worst row: {_worst_row(g, r)})"
    return max_abs, rel


def _worst_row(g, r):
    """Index and relative L2 error of the worst row along the last axis (for failure
    messages only)."""
    if r.ndim < 2 or r.size == 0:
        return None
    gg, rr = g.reshape(-1, r.shape[-1]), r.reshape(-1, r.shape[-1])
    ok = np.isfinite(rr).all(-1)
    if not ok.any():
        return None
    num = np.linalg.norm(gg - np.where(np.isfinite(rr), rr, 0), axis=-1)
    den = np.linalg.norm(np.where(np.isfinite(rr), rr, 0), axis=-1)
    rel = np.where(ok, num / np.where(den > 0, den, 1.0), -1.0)
    row = int(np.argmax(rel))
    return tuple(int(x) for x in np.unravel_index(row, r.shape[:-1])), float(rel[row])


def assert_same_selection(idx_gpu, nsel_gpu, idx_ref, nsel_ref, what=""):
    """Bit-exact comparison of kept chunk lists (both in ascending chunk index)."""
    ig = host(idx_gpu).numpy()
    ng = host(nsel_gpu).numpy()
    assert (ng == np.asarray(nsel_ref)).all(), f"{what}: nsel differs"
    bad = np.argwhere((ig != np.asarray(idx_ref)).any(-1))
    assert bad.size == 0, f"{what}: {len(bad)} selection rows differ, first {bad[:3].tolist()}"


def scores_close(score_gpu, score_ref, nsel, what=""):
    """float32 screen scores against the float64 values, within 1e-5 + 2e-6 |s|."""
    g = host(score_gpu).double().numpy()
    r = np.asarray(score_ref, np.float64)
    kept = np.arange(g.shape[-1]) < np.asarray(nsel)[..., None]
    err = np.abs(g[kept] - r[kept])
    tol = 1e-5 + 2e-6 * np.abs(r[kept])
    assert (err <= tol).all(), f"{what}: score err {float(err.max()):.3e}"
    assert np.isneginf(g[~kept]).all(), f"{what}: padding is not -inf"
