"""Pins of the oracle's window-exclusion variant (the `HILS_FLAG_EXCLUDE_WINDOW_CHUNKS`
flag of the library): a chunk lying wholly inside the query's sliding window is not
eligible for selection, because the window attends its tokens exactly ("Hierarchical
Sparse Attention Done Right", summary page, Methodology 2: one normaliser over the
selected chunks and the window; the pages do not say whether a chunk may be counted in
both). Each pin ties the variant to something other than itself: the eligibility rule
restated from its definition over the plain scores, the reduction to the plain
selection at W = 0, and, for windows that start on a chunk boundary, exact causal
softmax attention over all tokens."""
import numpy as np
import pytest
import torch

import oracle

S = 64


def _rand(*shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g) * scale


def _inputs(B=1, H=2, Lq=40, d=16, C=30, seed=0):
    Qcal = _rand(B, H, Lq, d, seed=seed + 1)
    Ksum = _rand(B, H, C, d, seed=seed + 2, scale=0.5)
    Bsum = _rand(B, H, C, seed=seed + 3, scale=0.2)
    return Qcal, Ksum, Bsum


def test_zero_window_changes_nothing():
    Qcal, Ksum, Bsum = _inputs()
    qpos = torch.tensor([[64 * 7 + 5 * i for i in range(40)]], dtype=torch.int32)
    a = oracle.select(Qcal, Ksum, Bsum, S, 5, 0.3, qpos=qpos)
    b = oracle.select(Qcal, Ksum, Bsum, S, 5, 0.3, qpos=qpos, exclude_window=0)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("W", [1, 64, 100, 128, 700, 5000])
def test_selection_is_the_plain_ranking_over_chunks_starting_before_the_window(W):
    """Brute force: eligible = complete chunks before the query's own chunk that start
    before the window's first token max(0, t - W + 1); rank the plain Eq. 7 scores."""
    Qcal, Ksum, Bsum = _inputs(H=3, Lq=37, C=41, seed=10)
    K = 6
    qpos = torch.tensor([[64 * 3 + 97 * i for i in range(37)]], dtype=torch.int32)
    idx, score, nsel = oracle.select(Qcal, Ksum, Bsum, S, K, 0.25, qpos=qpos, exclude_window=W)
    plain = oracle.score_all(Qcal, Ksum, Bsum, S, 0.25, qpos=qpos)  # no exclusion
    for h in range(3):
        for i in range(37):
            t = int(qpos[0, i])
            w0 = max(0, t - W + 1)
            elig = [c for c in range(41) if c < t // S and c * S < w0]
            order = sorted(elig, key=lambda c: (-plain[0, h, i, c], c))
            keep = sorted(order[:K])
            assert nsel[0, h, i] == len(keep)
            assert list(idx[0, h, i, :len(keep)]) == keep
            assert np.array_equal(score[0, h, i, :len(keep)], plain[0, h, i, keep])
    # the variant's own score table marks exactly the excluded chunks -inf
    excl = oracle.score_all(Qcal, Ksum, Bsum, S, 0.25, qpos=qpos, exclude_window=W)
    for i in range(37):
        t = int(qpos[0, i])
        w0 = max(0, t - W + 1)
        for c in range(41):
            ok = c < t // S and c * S < w0
            assert np.isfinite(excl[0, :, i, c]).all() == ok


def test_window_covering_every_chunk_leaves_nothing_to_select():
    Qcal, Ksum, Bsum = _inputs(Lq=20)
    qpos = torch.tensor([[64 * 2 + 31 * i for i in range(20)]], dtype=torch.int32)
    W = int(qpos.max()) + 1
    _, _, nsel = oracle.select(Qcal, Ksum, Bsum, S, 4, 0.3, qpos=qpos, exclude_window=W)
    assert (nsel == 0).all()


def test_chunk_aligned_window_gives_exact_causal_attention():
    """Window start on a chunk boundary, every eligible chunk kept with its exact log-mass
    as score: the kept chunks and the window partition the tokens [0, t] with no overlap
    and no gap, so Eq. 10 is plain causal softmax attention over all of them."""
    B, H, N, d, W = 1, 2, 64 * 12, 16, 192
    Q = _rand(B, H, N, d, seed=21, scale=0.5)
    Kc = _rand(B, H, N, d, seed=22, scale=0.5)
    Vc = _rand(B, H, N, d, seed=23)
    # queries at the last token of a chunk: t + 1 - W is a multiple of 64
    ts = [64 * m - 1 for m in range(4, 13)]
    Lq = len(ts)
    qpos = torch.tensor([ts], dtype=torch.int32)
    Qq = Q[:, :, ts].contiguous()
    K = 12
    idx = np.full((B, H, Lq, K), -1, np.int32)
    nsel = np.zeros((B, H, Lq), np.int32)
    for i, t in enumerate(ts):
        w0 = max(0, t - W + 1)
        n = min(t // S, (w0 + S - 1) // S)  # the variant's eligible count
        idx[:, :, i, :n] = np.arange(n)
        nsel[:, :, i] = n
    # the selection the variant makes when every eligible chunk fits
    Qcal = _rand(B, H, Lq, d, seed=24)
    Ksum = _rand(B, H, 12, d, seed=25)
    Bsum = _rand(B, H, 12, seed=26)
    i2, _, n2 = oracle.select(Qcal, Ksum, Bsum, S, K, 0.25, qpos=qpos, exclude_window=W)
    assert np.array_equal(i2, idx) and np.array_equal(n2, nsel)
    score = oracle.chunk_logmass(Qq, Kc, idx, nsel, S, 0.25)
    O, lse = oracle.attend(Qq, Kc, Vc, idx, score, nsel, S, W, 0.25, qpos=qpos)
    Qd, Kd, Vd = (x[0].double().numpy() for x in (Qq, Kc, Vc))
    for h in range(H):
        for i, t in enumerate(ts):
            lg = Kd[h, : t + 1] @ Qd[h, i] * 0.25
            p = np.exp(lg - lg.max())
            ref = (p / p.sum()) @ Vd[h, : t + 1]
            assert np.abs(O[0, h, i] - ref).max() < 1e-12
            assert abs(lse[0, h, i] - (lg.max() + np.log(p.sum()))) < 1e-12
