"""Pins of the backward oracle (``oracle/backward.py``): its forward against the pinned C
oracle, and its autograd gradients against central finite differences (float64
``torch.autograd.gradcheck``), for multi-head and grouped heads, with and without a
window, so that a wrong term of the backward cannot pass."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob

S = 64


def _rand(*shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float64) * scale)


def _selection(B, Hk, N, K, seed):
    """A random valid selection: for query i, K distinct eligible chunks (c < i // 64)."""
    g = np.random.default_rng(seed)
    idx = np.full((B, Hk, N, K), -1, np.int32)
    nsel = np.zeros((B, Hk, N), np.int32)
    for b in range(B):
        for h in range(Hk):
            for i in range(N):
                ne = i // S
                n = min(K, ne)
                if n:
                    idx[b, h, i, :n] = np.sort(g.choice(ne, n, replace=False))
                nsel[b, h, i] = n
    return idx, nsel


def _problem(B=1, H=2, G=1, N=64 * 4 + 9, d=8, K=2, seed=0):
    Hk = H // G
    C = N // S
    Q = _rand(B, H, N, d, seed=seed + 1, scale=0.6)
    Kc = _rand(B, Hk, N, d, seed=seed + 2, scale=0.6)
    Vc = _rand(B, Hk, N, d, seed=seed + 3)
    Qcal = _rand(B, H, N, d, seed=seed + 4, scale=0.6)
    LQ = _rand(B, H, C, d, seed=seed + 5, scale=0.6)
    idx, nsel = _selection(B, Hk, N, K, seed + 6)
    return Q, Kc, Vc, Qcal, LQ, idx, nsel


@pytest.mark.parametrize("G,W", [(1, 40), (2, 70), (1, 0)])
def test_forward_matches_the_c_oracle(G, W):
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=4, G=G, N=64 * 5 + 17, d=16, K=3, seed=10)
    O, lse, score, Ksum, Bsum = ob.forward(Q, Kc, Vc, Qcal, LQ, idx, nsel, S, W, 0.3)
    ks, bs = oracle.summarize(Kc, LQ, S, 0.3)
    assert np.abs(Ksum.numpy() - ks).max() < 1e-12 and np.abs(Bsum.numpy() - bs).max() < 1e-12
    sall = oracle.score_all(Qcal, torch.from_numpy(ks), torch.from_numpy(bs), S, 0.3)
    Hk = Kc.shape[1]
    for h in range(4):
        for i in range(Q.shape[2]):
            n = nsel[0, h // G, i]
            cs = idx[0, h // G, i, :n]
            if n:
                assert np.abs(score[0, h, i, :n].numpy() - sall[0, h, i, cs]).max() < 1e-12
            assert np.isneginf(score[0, h, i, n:].numpy()).all()
    O_ref, lse_ref = oracle.attend(Q, Kc, Vc, idx, score.numpy(), nsel, S, W, 0.3)
    assert np.abs(O.numpy() - O_ref).max() < 1e-12
    fin = np.isfinite(lse_ref)
    assert (np.isfinite(lse.numpy()) == fin).all()
    assert np.abs(lse.numpy()[fin] - lse_ref[fin]).max() < 1e-12
    assert Hk * G == 4


@pytest.mark.parametrize("G,W", [(1, 30), (2, 70), (1, 0)])
def test_gradients_match_finite_differences(G, W):
    """float64 gradcheck of every input's gradient (central differences, eps 1e-6; the
    fast mode checks the gradients along random directions of every input)."""
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=2, G=G, N=64 * 3 + 5, d=4, K=2, seed=20 + G)
    dO = _rand(*Q.shape, seed=99)

    def f(q, k, v, qc, lq):
        O, _, _, _, _ = ob.forward(q, k, v, qc, lq, idx, nsel, S, W, 0.4)
        return (O * dO).sum()

    ins = [x.clone().requires_grad_(True) for x in (Q, Kc, Vc, Qcal, LQ)]
    assert torch.autograd.gradcheck(f, ins, eps=1e-6, atol=1e-7, rtol=1e-5, fast_mode=True)
    # the grads() wrapper returns the same gradients
    g = ob.grads(Q, Kc, Vc, Qcal, LQ, idx, nsel, dO, S, W, 0.4)
    auto = torch.autograd.grad(f(*ins), ins)
    for name, a in zip(("dQ", "dK", "dV", "dQcal", "dLQ"), auto):
        assert torch.allclose(g[name], a, atol=1e-14, rtol=0), name


def test_intermediate_gradients_by_the_chain_rule():
    """dscore, dKsum, dBsum against their closed forms from the other gradients:
    dQcal = scale sum_k dscore_k k'_{c_k}; dBsum_c = sum over the queries that kept c
    of dscore; dKsum_c = scale sum of dscore q~."""
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=2, G=1, N=64 * 4 + 3, d=8, K=3, seed=30)
    dO = _rand(*Q.shape, seed=31)
    g = ob.grads(Q, Kc, Vc, Qcal, LQ, idx, nsel, dO, S, 50, 0.35)
    _, _, _, Ksum, Bsum = ob.forward(Q, Kc, Vc, Qcal, LQ, idx, nsel, S, 50, 0.35)
    B, H, N, d = Q.shape
    dq = torch.zeros_like(Qcal)
    dks = torch.zeros_like(Ksum)
    dbs = torch.zeros_like(Bsum)
    for h in range(H):
        for i in range(N):
            for k in range(int(nsel[0, h, i])):
                c = int(idx[0, h, i, k])
                ds = g["dscore"][0, h, i, k]
                dq[0, h, i] += 0.35 * ds * Ksum[0, h, c].detach()
                dks[0, h, c] += 0.35 * ds * Qcal[0, h, i]
                dbs[0, h, c] += ds
    assert torch.allclose(g["dQcal"], dq, atol=1e-12)
    assert torch.allclose(g["dKsum"], dks, atol=1e-12)
    assert torch.allclose(g["dBsum"], dbs, atol=1e-12)


def test_gradients_match_finite_differences_elementwise():
    """The full (element by element) float64 gradcheck on a small case: two chunks, a
    window crossing a chunk boundary, two query heads sharing a key-value head."""
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=2, G=2, N=64 * 2 + 7, d=2, K=1, seed=40)
    dO = _rand(*Q.shape, seed=41)

    def f(q, k, v, qc, lq):
        O, _, _, _, _ = ob.forward(q, k, v, qc, lq, idx, nsel, S, 20, 0.5)
        return (O * dO).sum()

    ins = [x.clone().requires_grad_(True) for x in (Q, Kc, Vc, Qcal, LQ)]
    assert torch.autograd.gradcheck(f, ins, eps=1e-6, atol=1e-7, rtol=1e-5)


@pytest.mark.parametrize("G,W,batch", [(1, 60, 50), (2, 90, 64), (1, 0, 7)])
def test_row_blocks_give_the_same_gradients(G, W, batch):
    """The row-block form used at long sequences: forward over a subset of rows equals
    those rows of the full forward, and gradients summed over row blocks (a block size
    that does not divide N) equal the gradients of the whole problem."""
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=2, G=G, N=64 * 4 + 21, d=8, K=3, seed=50 + G)
    dO = _rand(*Q.shape, seed=51)
    full = ob.grads(Q, Kc, Vc, Qcal, LQ, idx, nsel, dO, S, W, 0.45)
    blk = ob.grads(Q, Kc, Vc, Qcal, LQ, idx, nsel, dO, S, W, 0.45, batch=batch)
    for name in ("dQ", "dK", "dV", "dQcal", "dLQ", "dscore", "dKsum", "dBsum", "O"):
        assert torch.allclose(blk[name], full[name], atol=1e-12, rtol=0), name
    fin = torch.isfinite(full["lse"])
    assert torch.equal(torch.isfinite(blk["lse"]), fin)
    assert torch.allclose(blk["lse"][fin], full["lse"][fin], atol=1e-12, rtol=0)
    rows = np.array([0, 5, 64, 65, 200, Q.shape[2] - 1])
    O, lse, score, _, _ = ob.forward(Q, Kc, Vc, Qcal, LQ, idx, nsel, S, W, 0.45, rows=rows)
    assert torch.allclose(O, full["O"][:, :, rows], atol=1e-12, rtol=0)


def test_key_value_head_slices_are_independent_problems():
    """Each key-value head with its G query heads is a problem of its own: the gradients
    of a slice computed alone equal that slice of the whole problem's gradients (the
    form the full-size GPU test compares on)."""
    G = 2
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=4, G=G, N=64 * 3 + 11, d=8, K=2, seed=60)
    dO = _rand(*Q.shape, seed=61)
    full = ob.grads(Q, Kc, Vc, Qcal, LQ, idx, nsel, dO, S, 80, 0.5)
    hk = 1
    qs, ks = slice(hk * G, (hk + 1) * G), slice(hk, hk + 1)
    part = ob.grads(Q[:, qs], Kc[:, ks], Vc[:, ks], Qcal[:, qs], LQ[:, qs], idx[:, ks], nsel[:, ks], dO[:, qs], S, 80,
                    0.5, batch=64)
    for name in ("dQ", "dQcal", "dLQ", "dscore", "dKsum", "dBsum"):
        assert torch.allclose(part[name], full[name][:, qs], atol=1e-12, rtol=0), name
    for name in ("dK", "dV"):
        assert torch.allclose(part[name], full[name][:, ks], atol=1e-12, rtol=0), name


@pytest.mark.parametrize("G,W", [(1, 50), (2, 90)])
def test_value_gradients_sum_to_the_output_gradients(G, W):
    """Eq. 10 gives every query one normaliser over its kept chunks and its window, so
    the token weights of a query with a finite lse sum to 1 and dO_i reaches the values
    with total weight 1: for each key-value head, sum_j dV_j = sum of dO_i over its
    query heads' queries (all of them here: W > 0 puts each query's own token in its
    window). Independent of autograd: a wrong weight or a dropped term breaks it."""
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=4, G=G, N=64 * 4 + 29, d=8, K=3, seed=70 + G)
    dO = _rand(*Q.shape, seed=71)
    g = ob.grads(Q, Kc, Vc, Qcal, LQ, idx, nsel, dO, S, W, 0.4)
    assert torch.isfinite(g["lse"]).all()
    want = dO.reshape(1, 4 // G, G, *dO.shape[2:]).sum(dim=(2, 3))  # [B, Hk, d]
    assert torch.allclose(g["dV"].sum(dim=2), want, atol=1e-11, rtol=0)


def test_score_gradient_closed_form():
    """dscore against its closed form from Eq. 10, with every ingredient from the C
    oracle rather than autograd: for query i and kept chunk c, with w_c = exp(s^_c -
    lse_i), o_c the chunk's own softmax average of its values, and D_i = dO_i . o_i,
    the gradient of sum(O * dO) with respect to s^_c is w_c (dO_i . o_c - D_i)."""
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=2, G=1, N=64 * 4 + 13, d=8, K=3, seed=80)
    dO = _rand(*Q.shape, seed=81)
    W, sc = 45, 0.5
    g = ob.grads(Q, Kc, Vc, Qcal, LQ, idx, nsel, dO, S, W, sc)
    ks, bs = oracle.summarize(Kc, LQ, S, sc)
    sall = oracle.score_all(Qcal, torch.from_numpy(ks), torch.from_numpy(bs), S, sc)
    score = np.full(idx.shape, -np.inf)
    for h in range(2):
        for i in range(Q.shape[2]):
            n = nsel[0, h, i]
            score[0, h, i, :n] = sall[0, h, i, idx[0, h, i, :n]]
    O, lse = oracle.attend(Q, Kc, Vc, idx, score, nsel, S, W, sc)
    q, k, v, do = (x.numpy() for x in (Q, Kc, Vc, dO))
    want = np.zeros(idx.shape)
    for h in range(2):
        for i in range(Q.shape[2]):
            Di = do[0, h, i] @ O[0, h, i]
            for slot in range(nsel[0, h, i]):
                c = idx[0, h, i, slot]
                lg = sc * (k[0, h, c * S:(c + 1) * S] @ q[0, h, i])
                p = np.exp(lg - lg.max())
                oc = (p / p.sum()) @ v[0, h, c * S:(c + 1) * S]
                want[0, h, i, slot] = np.exp(score[0, h, i, slot] - lse[0, h, i]) * (do[0, h, i] @ oc - Di)
    assert np.abs(g["dscore"].numpy() - want).max() < 1e-12
    assert (nsel > 0).any() and (nsel < 3).any()


def test_empty_queries_pass_no_gradient():
    """With W = 0, the first 64 queries keep no chunk and have an empty window: o = 0 and
    lse = -inf, a constant output, so their dQ, dQcal and dscore are exactly 0 and no
    gradient is NaN anywhere."""
    Q, Kc, Vc, Qcal, LQ, idx, nsel = _problem(H=2, G=1, N=64 * 3 + 7, d=8, K=2, seed=90)
    dO = _rand(*Q.shape, seed=91)
    g = ob.grads(Q, Kc, Vc, Qcal, LQ, idx, nsel, dO, S, 0, 0.5)
    assert torch.isneginf(g["lse"][..., :64]).all() and torch.isfinite(g["lse"][..., 64:]).all()
    for name in ("dQ", "dQcal", "dscore"):
        assert (g[name][:, :, :64] == 0).all(), name
    for name in ("dQ", "dK", "dV", "dQcal", "dLQ", "dscore", "dKsum", "dBsum"):
        assert torch.isfinite(g[name]).all(), name
    assert (g["O"][:, :, :64] == 0).all()
