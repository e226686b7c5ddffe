"""Pins of the oracle's grouped-query attention ("Hierarchical Sparse Attention Done
Right", summary page, Methodology 3, GQA adaptation: the heads of a group keep the chunks
with the largest maximum of their chunk scores). Each pin ties the grouped routines to
something other than themselves: the identity with multi-head attention over repeated
key-value heads, the special cases where the maximum is one head's score, and a
brute-force ranking of the per-head scores."""
import numpy as np
import pytest
import torch

import oracle

S = 64


def _rand(*shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g) * scale


def _rank_topk(group_scores: np.ndarray, K: int):
    """Brute force: sort by (score descending, index ascending), keep K, list ascending."""
    order = sorted(range(len(group_scores)), key=lambda c: (-group_scores[c], c))
    keep = sorted(order[:K])
    return keep


@pytest.mark.parametrize("G", [2, 4])
def test_grouped_summaries_equal_multihead_over_repeated_kv(G):
    B, Hk, N, d = 1, 2, 64 * 5 + 7, 32
    H = Hk * G
    K = _rand(B, Hk, N, d, seed=1)
    LQ = _rand(B, H, N // S, d, seed=2)
    ks, bs = oracle.summarize(K, LQ, S, 0.25)
    ks1, bs1 = oracle.summarize(K.repeat_interleave(G, dim=1).contiguous(), LQ, S, 0.25)
    assert np.array_equal(ks, ks1) and np.array_equal(bs, bs1)


@pytest.mark.parametrize("G,K", [(2, 3), (3, 4), (4, 1)])
def test_grouped_selection_brute_force(G, K):
    """Group score = max over heads of s^ (from score_all, pinned on its own); top K by
    (score desc, index asc), ascending; each head reports its own s^ of the kept chunks."""
    B, Hk, Lq, d, C = 2, 2, 9, 16, 11
    H = Hk * G
    Qcal = _rand(B, H, Lq, d, seed=3)
    Ksum = _rand(B, H, C, d, seed=4, scale=0.5)
    Bsum = _rand(B, H, C, seed=5, scale=0.2)
    qpos = torch.tensor([[64 * c + 13 for c in range(Lq)]] * B, dtype=torch.int32)  # 0..8 eligible
    idx, score, nsel = oracle.select(Qcal, Ksum, Bsum, S, K, 0.3, qpos=qpos, group=G)
    assert idx.shape == (B, Hk, Lq, K) and score.shape == (B, H, Lq, K) and nsel.shape == (B, Hk, Lq)
    sall = oracle.score_all(Qcal, Ksum, Bsum, S, 0.3, qpos=qpos)  # [B, H, Lq, C], -inf ineligible
    for b in range(B):
        for g in range(Hk):
            for i in range(Lq):
                grp = sall[b, g * G:(g + 1) * G, i]
                ne = int(np.isfinite(grp[0]).sum())
                keep = _rank_topk(grp.max(0)[:ne], K)
                assert nsel[b, g, i] == len(keep)
                assert list(idx[b, g, i, :len(keep)]) == keep
                assert (idx[b, g, i, len(keep):] == -1).all()
                for hh in range(G):
                    h = g * G + hh
                    assert np.array_equal(score[b, h, i, :len(keep)], sall[b, h, i, keep])
                    assert np.isneginf(score[b, h, i, len(keep):]).all()


def test_grouped_selection_reduces_to_multihead():
    """Identical heads inside each group: the group maximum is every head's own score, so
    the group keeps exactly the multi-head selection of any of its heads. One dominant
    head (bias + 1000): the group keeps that head's own selection."""
    B, Hk, G, Lq, d, C, K = 1, 3, 3, 20, 16, 40, 5
    H = Hk * G
    q1 = _rand(B, Hk, Lq, d, seed=6)
    k1 = _rand(B, Hk, C, d, seed=7, scale=0.5)
    b1 = _rand(B, Hk, C, seed=8, scale=0.1)
    rep = lambda x: x.repeat_interleave(G, dim=1).contiguous()  # noqa: E731
    qpos = torch.full((B, Lq), 64 * C + 5, dtype=torch.int32)
    idx, score, nsel = oracle.select(rep(q1), rep(k1), rep(b1), S, K, 0.25, qpos=qpos, group=G)
    i1, s1, n1 = oracle.select(q1, k1, b1, S, K, 0.25, qpos=qpos)
    assert np.array_equal(idx, i1) and np.array_equal(nsel, n1)
    assert np.array_equal(score, np.repeat(s1, G, axis=1))
    # one dominant head per group
    Qcal = _rand(B, H, Lq, d, seed=9)
    Ksum = _rand(B, H, C, d, seed=10, scale=0.5)
    Bsum = _rand(B, H, C, seed=11, scale=0.1).double()
    dom = [1, 0, 2]
    for g, hh in enumerate(dom):
        Bsum[:, g * G + hh] += 1000.0
    idx, score, nsel = oracle.select(Qcal, Ksum, Bsum, S, K, 0.25, qpos=qpos, group=G)
    for g, hh in enumerate(dom):
        h = g * G + hh
        ih, sh, nh = oracle.select(Qcal[:, h:h + 1], Ksum[:, h:h + 1], Bsum[:, h:h + 1], S, K, 0.25, qpos=qpos)
        assert np.array_equal(idx[:, g], ih[:, 0]) and np.array_equal(nsel[:, g], nh[:, 0])
        assert np.array_equal(score[:, h], sh[:, 0])


@pytest.mark.parametrize("G", [2, 4])
def test_grouped_attend_equals_multihead_over_repeated_kv(G):
    """Each query head reads its key-value head and its group's kept chunks: the output
    is multi-head attention over repeated key-value heads and repeated kept lists."""
    B, Hk, N, d, K, W = 1, 2, 64 * 6 + 9, 16, 3, 50
    H = Hk * G
    Q = _rand(B, H, N, d, seed=12, scale=0.5)
    Kc = _rand(B, Hk, N, d, seed=13, scale=0.5)
    Vc = _rand(B, Hk, N, d, seed=14)
    g = np.random.default_rng(15)
    idx = np.full((B, Hk, N, K), -1, np.int32)
    nsel = np.zeros((B, Hk, N), np.int32)
    for hk in range(Hk):
        for i in range(N):
            ne = min(i // S, N // S)
            n = min(K, ne)
            idx[0, hk, i, :n] = np.sort(g.choice(ne, n, replace=False)) if n else []
            nsel[0, hk, i] = n
    score = torch.from_numpy(g.normal(4.0, 0.5, (B, H, N, K)))
    O, lse = oracle.attend(Q, Kc, Vc, idx, score, nsel, S, W, 0.25)
    rep = lambda x: x.repeat_interleave(G, dim=1).contiguous()  # noqa: E731
    O1, lse1 = oracle.attend(Q, rep(Kc), rep(Vc), np.repeat(idx, G, axis=1), score, np.repeat(nsel, G, axis=1),
                             S, W, 0.25)
    assert np.array_equal(O, O1) and np.array_equal(lse, lse1)
