"""Pins of the float64 oracle against facts the pages and the mathematics fix.

The oracle is the parity reference for every GPU test, so it is checked here
against things other than itself:
  * hand-worked Eq. 8 cases with closed-form answers (tests/golden);
  * the Taylor identity of Eq. 7 at q = q'_c, and the tangent (convexity) bound;
  * the two log-Z regimes of the Introduction (uniform logits: mean + log S;
    one dominant logit: max);
  * brute-force enumeration of top-K subsets, with planted exact ties;
  * reductions of Eq. 10 to plain softmax attention computed by torch in float64.
Sources: "Hierarchical Sparse Attention Done Right" (picx.dev summary), Introduction,
Methodology 1 (Eq. 7, Eq. 8), Methodology 2 (Eq. 10); same title (rcap.io post),
pseudocode figure.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "eq8_worked_cases.txt")


def _rand(shape, seed, dtype=torch.float64, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale).to(dtype)


def _ln_eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"ln": math.log}))


def _golden_cases():
    cases, cur = [], None
    for raw in open(GOLDEN):
        line = raw.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest}
        elif key == "end":
            cases.append(cur)
            cur = None
        elif key in ("d", "S"):
            cur[key] = int(rest)
        elif key == "scale":
            cur[key] = _ln_eval(rest)
        elif key == "lq":
            cur[key] = [_ln_eval(v) for v in rest.split()]
        elif key == "keys":
            cur[key] = [[_ln_eval(v) for v in row.split()] for row in rest.split("|")]
        elif key == "ksum":
            cur[key] = [_ln_eval(v) for v in rest.split(";")]
        elif key in ("bsum", "logZ"):
            cur[key] = _ln_eval(rest)
    return cases


# ----------------------------------------------------------------- Eq. 8 summaries

@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_eq8_hand_worked_cases(oracle, case):
    d, S = case["d"], case["S"]
    K = torch.tensor(case["keys"], dtype=torch.float64).reshape(1, 1, S, d)
    LQ = torch.tensor(case["lq"], dtype=torch.float64).reshape(1, 1, 1, d)
    ksum, bsum = oracle.summarize(K, LQ, S, case["scale"])
    np.testing.assert_allclose(ksum[0, 0, 0], case["ksum"], rtol=0, atol=1e-14)
    assert abs(bsum[0, 0, 0] - case["bsum"]) < 1e-14
    # Eq. 7 at the Taylor point reproduces the exact log-mass of the chunk
    s = oracle.score_all(LQ, ksum, bsum, S, case["scale"], qpos=np.array([[S]]))
    assert abs(s[0, 0, 0, 0] - case["logZ"]) < 1e-14


def _summaries(seed, B=1, H=2, C=5, S=8, d=16, lq_scale=1.0):
    K = _rand((B, H, C * S, d), seed)
    LQ = _rand((B, H, C, d), seed + 1, scale=lq_scale)
    return K, LQ


def _exact_logmass(q, Kchunk, scale):
    return logsumexp(Kchunk.numpy() @ q.numpy() * scale)


def test_taylor_identity_at_landmark_query(oracle):
    """At q = q'_c the surrogate of Eq. 7 equals log Z_c exactly (the expansion point)."""
    S, d, C = 8, 16, 5
    scale = 1 / math.sqrt(d)
    K, LQ = _summaries(11, C=C, S=S, d=d)
    ksum, bsum = oracle.summarize(K, LQ, S, scale)
    # query i = q'_i, placed late enough that every chunk is eligible
    qpos = np.full((1, C), C * S, np.int32)
    s = oracle.score_all(LQ, ksum, bsum, S, scale, qpos=qpos)
    for h in range(2):
        for c in range(C):
            ref = _exact_logmass(LQ[0, h, c], K[0, h, c * S:(c + 1) * S], scale)
            assert abs(s[0, h, c, c] - ref) < 1e-12


def test_surrogate_is_a_tangent_lower_bound(oracle):
    """log Z_c(q) is convex in q and Eq. 7 is its tangent at q'_c: s^_c(q) <= log Z_c(q)."""
    S, d, C = 8, 16, 5
    scale = 1 / math.sqrt(d)
    K, LQ = _summaries(21, C=C, S=S, d=d)
    ksum, bsum = oracle.summarize(K, LQ, S, scale)
    Q = _rand((1, 2, 40, d), 22, scale=2.0)
    s = oracle.score_all(Q, ksum, bsum, S, scale, qpos=np.full((1, 40), C * S, np.int32))
    gap_max = 0.0
    for h in range(2):
        for i in range(40):
            for c in range(C):
                ref = _exact_logmass(Q[0, h, i], K[0, h, c * S:(c + 1) * S], scale)
                assert s[0, h, i, c] <= ref + 1e-12
                gap_max = max(gap_max, ref - s[0, h, i, c])
    assert gap_max > 1e-3  # the bound is not trivially tight away from q'


def test_uniform_regime(oracle):
    """Equal keys in a chunk: log Z = scale q.k + log S, and Eq. 7 is exact for every q.
    With q' = 0 the landmark softmax is uniform: b' = log S and k' = mean of the keys."""
    S, d = 8, 16
    scale = 1 / math.sqrt(d)
    k = _rand((d,), 31)
    K = k.repeat(1, 1, S, 1)  # [1,1,S,d], every row = k
    LQ = _rand((1, 1, 1, d), 32)
    ksum, bsum = oracle.summarize(K, LQ, S, scale)
    assert abs(bsum[0, 0, 0] - math.log(S)) < 1e-13
    np.testing.assert_allclose(ksum[0, 0, 0], k.numpy(), rtol=0, atol=1e-14)
    Q = _rand((1, 1, 7, d), 33)
    s = oracle.score_all(Q, ksum, bsum, S, scale, qpos=np.full((1, 7), S, np.int32))
    for i in range(7):
        want = float(Q[0, 0, i] @ k) * scale + math.log(S)
        assert abs(s[0, 0, i, 0] - want) < 1e-12

    K2 = _rand((1, 1, S, d), 34)
    ksum2, bsum2 = oracle.summarize(K2, torch.zeros(1, 1, 1, d, dtype=torch.float64), S, scale)
    assert abs(bsum2[0, 0, 0] - math.log(S)) < 1e-13
    np.testing.assert_allclose(ksum2[0, 0, 0], K2[0, 0].mean(0).numpy(), rtol=0, atol=1e-14)


def test_dominant_regime(oracle):
    """q' = lam * k_j* with large lam: p concentrates on j*, so b' -> 0, k' -> k_j*, and the
    surrogate tends to the max logit; always max <= log Z <= max + log S."""
    S, d = 8, 16
    scale = 1 / math.sqrt(d)
    K = _rand((1, 1, S, d), 41)
    jstar = 5
    LQ = (K[0, 0, jstar] * 400.0).reshape(1, 1, 1, d)
    ksum, bsum = oracle.summarize(K, LQ, S, scale)
    assert 0.0 <= bsum[0, 0, 0] < 1e-9
    np.testing.assert_allclose(ksum[0, 0, 0], K[0, 0, jstar].numpy(), rtol=0, atol=1e-9)
    Q = _rand((1, 1, 9, d), 42)
    for i in range(9):
        logits = K[0, 0].numpy() @ Q[0, 0, i].numpy() * scale
        lz = logsumexp(logits)
        assert logits.max() <= lz <= logits.max() + math.log(S) + 1e-12
    # at the expansion point the surrogate is log Z itself, which is ~ the max logit
    s = oracle.score_all(LQ, ksum, bsum, S, scale, qpos=np.array([[S]], np.int32))
    lg = K[0, 0].numpy() @ LQ[0, 0, 0].numpy() * scale
    assert abs(s[0, 0, 0, 0] - lg.max()) < 1e-9


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float64])
def test_summary_bounds(oracle, dtype):
    """0 <= b' <= log S (entropy of S outcomes) and k' lies in the keys' convex hull."""
    S, d, C = 64, 64, 6
    K = _rand((2, 3, C * S, d), 51, dtype=dtype)
    LQ = _rand((2, 3, C, d), 52, dtype=dtype, scale=3.0)
    ksum, bsum = oracle.summarize(K, LQ, S, 1 / 8)
    assert (bsum >= 0).all() and (bsum <= math.log(S) + 1e-12).all()
    Kd = K.double().reshape(2, 3, C, S, d).numpy()
    assert (ksum <= Kd.max(3) + 1e-12).all() and (ksum >= Kd.min(3) - 1e-12).all()


def test_summary_reads_strided_views(oracle):
    """A non-contiguous [B,H,N,d] view reads the same elements as its contiguous copy."""
    S, d = 8, 16
    base = _rand((1, 5, 3 * S, d), 61).permute(1, 0, 2, 3)  # [5,1,N,d], batch stride != H*N*d
    LQ = _rand((5, 1, 3, d), 62)
    a = oracle.summarize(base, LQ, S, 0.25)
    b = oracle.summarize(base.contiguous(), LQ, S, 0.25)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


# ------------------------------------------------------------------ scores and top-K

def test_scores_match_a_library_matmul(oracle):
    """Eq. 7 with q~: the oracle's ordered sum agrees with a float64 matmul to rounding."""
    S, d, C, Lq = 8, 32, 10, 12
    Qc = _rand((1, 2, Lq, d), 71)
    ks = _rand((1, 2, C, d), 72)
    bs = _rand((1, 2, C), 73).abs()
    scale = 1 / math.sqrt(d)
    s = oracle.score_all(Qc, ks, bs, S, scale, qpos=np.full((1, Lq), C * S, np.int32))
    ref = (Qc @ ks.transpose(-1, -2)).numpy() * scale + bs.numpy()[:, :, None, :]
    np.testing.assert_allclose(s, ref, rtol=1e-13, atol=1e-13)


def _brute_topk(scores, K):
    """Best K-subset by exact sum; among equal sums the lexicographically smallest."""
    n = len(scores)
    best, best_sum = None, None
    for sub in itertools.combinations(range(n), min(K, n)):
        tot = math.fsum(scores[list(sub)])
        if best is None or tot > best_sum or (tot == best_sum and sub < best):
            best, best_sum = sub, tot
    return list(best)


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_subset_enumeration(oracle, seed):
    rng = np.random.default_rng(seed)
    S, d = 4, 8
    C = int(rng.integers(3, 11))
    K = int(rng.integers(1, 5))
    Lq = 6
    Qc = _rand((1, 1, Lq, d), 100 + seed)
    ks = _rand((1, 1, C, d), 200 + seed)
    bs = _rand((1, 1, C), 300 + seed).abs()
    # plant exact ties: duplicate a chunk's summary into a later slot
    if C >= 4:
        ks[0, 0, C - 1] = ks[0, 0, 1]
        bs[0, 0, C - 1] = bs[0, 0, 1]
    qpos = rng.integers(0, (C + 2) * S, size=(1, Lq)).astype(np.int32)
    qpos[0, 0] = C * S  # at least one query sees every chunk
    idx, score, nsel = oracle.select(Qc, ks, bs, S, K, 0.5, qpos=qpos)
    all_s = oracle.score_all(Qc, ks, bs, S, 0.5, qpos=qpos)
    for i in range(Lq):
        ne = min(qpos[0, i] // S, C)
        want = sorted(_brute_topk(all_s[0, 0, i, :ne], K)) if ne else []
        n = int(nsel[0, 0, i])
        assert n == min(K, ne)
        assert list(idx[0, 0, i, :n]) == want
        assert (idx[0, 0, i, n:] == -1).all() and np.isneginf(score[0, 0, i, n:]).all()
        np.testing.assert_array_equal(score[0, 0, i, :n], all_s[0, 0, i, want])


def test_exact_tie_prefers_lower_chunk(oracle):
    S, d = 4, 8
    ks = _rand((1, 1, 6, d), 401)
    bs = torch.zeros(1, 1, 6, dtype=torch.float64)
    for c in (2, 4, 5):
        ks[0, 0, c] = ks[0, 0, 0]
    q = ks[0, 0, 0].reshape(1, 1, 1, d) * 10  # chunks 0, 2, 4, 5 tie for the top score
    idx, _, nsel = oracle.select(q, ks, bs, S, 3, 1.0, qpos=np.array([[6 * S]], np.int32))
    assert list(idx[0, 0, 0]) == [0, 2, 4] and nsel[0, 0, 0] == 3


def test_eligibility_excludes_own_and_partial_chunk(oracle):
    """Only complete chunks strictly before the query's own chunk are eligible."""
    S, d, C = 4, 8, 5
    ks = _rand((1, 1, C, d), 501)
    bs = torch.zeros(1, 1, C, dtype=torch.float64)
    pos = np.array([[0, 3, 4, 7, 8, 19, 20, 50]], np.int32)
    q = _rand((1, 1, pos.shape[1], d), 502)
    idx, _, nsel = oracle.select(q, ks, bs, S, C, 1.0, qpos=pos)
    assert list(nsel[0, 0]) == [0, 0, 1, 1, 2, 4, 5, 5]
    for i in range(pos.shape[1]):
        assert list(idx[0, 0, i, :nsel[0, 0, i]]) == list(range(nsel[0, 0, i]))


# ------------------------------------------------------------ Eq. 10 and reductions

def _causal_attention(q, K, V, lo, hi, scale):
    """Textbook softmax attention of q over keys [lo, hi] (float64 torch)."""
    logits = (K[lo:hi + 1] @ q) * scale
    w = torch.softmax(logits, 0)
    return (w @ V[lo:hi + 1]).numpy(), float(torch.logsumexp(logits, 0))


def test_exact_mass_with_every_chunk_is_full_attention_over_the_chunks(oracle):
    """Top-K = all eligible chunks, W = 0, chunk scores = exact log Z_{i,c}: Eq. 10 reduces
    to softmax attention over the keys of the complete chunks before the query's own."""
    S, d, N = 8, 16, 64
    C = N // S
    scale = 1 / math.sqrt(d)
    Q, K, V = _rand((1, 2, N, d), 601), _rand((1, 2, N, d), 602), _rand((1, 2, N, d), 603)
    idx = np.full((1, 2, N, C), -1, np.int32)
    nsel = np.zeros((1, 2, N), np.int32)
    for i in range(N):
        ne = i // S
        idx[:, :, i, :ne] = np.arange(ne)
        nsel[:, :, i] = ne
    score = oracle.chunk_logmass(Q, K, idx, nsel, S, scale)
    O, lse = oracle.attend(Q, K, V, idx, score, nsel, S, 0, scale)
    for h in range(2):
        for i in range(N):
            ne = i // S
            if ne == 0:
                assert (O[0, h, i] == 0).all() and np.isneginf(lse[0, h, i])
                continue
            o, l = _causal_attention(Q[0, h, i], K[0, h], V[0, h], 0, ne * S - 1, scale)
            np.testing.assert_allclose(O[0, h, i], o, rtol=0, atol=1e-12)
            assert abs(lse[0, h, i] - l) < 1e-12


def test_chunk_size_one_surrogate_path_is_exact_causal_attention(oracle):
    """S = 1: every chunk is one token, so k' = k, b' = 0 and Eq. 7 is exact. With q~ = q,
    K = all chunks and W = 1 (the query's own token), the whole surrogate path (summarise,
    select, attend) is exact full causal attention."""
    d, N = 16, 40
    scale = 1 / math.sqrt(d)
    Q, K, V = _rand((1, 1, N, d), 701), _rand((1, 1, N, d), 702), _rand((1, 1, N, d), 703)
    LQ = _rand((1, 1, N, d), 704)
    ksum, bsum = oracle.summarize(K, LQ, 1, scale)
    np.testing.assert_allclose(ksum, K.numpy(), rtol=0, atol=0)
    assert (bsum == 0).all()
    idx, score, nsel = oracle.select(Q, ksum, bsum, 1, N, scale)
    O, lse = oracle.attend(Q, K, V, idx, score, nsel, 1, 1, scale)
    for i in range(N):
        o, l = _causal_attention(Q[0, 0, i], K[0, 0], V[0, 0], 0, i, scale)
        np.testing.assert_allclose(O[0, 0, i], o, rtol=0, atol=1e-12)
        assert abs(lse[0, 0, i] - l) < 1e-12


@pytest.mark.parametrize("W", [1, 5, 64, 1000])
def test_window_only_is_local_causal_attention(oracle, W):
    S, d, N = 8, 16, 48
    scale = 1 / math.sqrt(d)
    Q, K, V = _rand((1, 1, N, d), 801), _rand((1, 1, N, d), 802), _rand((1, 1, N, d), 803)
    idx = np.full((1, 1, N, 2), -1, np.int32)
    nsel = np.zeros((1, 1, N), np.int32)
    score = np.full((1, 1, N, 2), -np.inf)
    O, lse = oracle.attend(Q, K, V, idx, score, nsel, S, W, scale)
    for i in range(N):
        o, l = _causal_attention(Q[0, 0, i], K[0, 0], V[0, 0], max(0, i - W + 1), i, scale)
        np.testing.assert_allclose(O[0, 0, i], o, rtol=0, atol=1e-12)
        assert abs(lse[0, 0, i] - l) < 1e-12


def test_empty_selection_and_window(oracle):
    Q = _rand((1, 1, 3, 8), 901)
    O, lse = oracle.attend(Q, Q, Q, np.full((1, 1, 3, 1), -1, np.int32),
                           np.full((1, 1, 3, 1), -np.inf), np.zeros((1, 1, 3), np.int32), 4, 0, 1.0)
    assert (O == 0).all() and np.isneginf(lse).all()


@pytest.mark.parametrize("seed", range(3))
def test_token_level_weights_sum_to_one_and_reproduce_output(oracle, seed):
    """Eq. 10 written per token: w_ij = e^{s_ij}/Z_{i,c(j)} * Z^_{i,c(j)}/Z^_i (+ window term)
    sums to one, and w . V equals the chunk-level combination."""
    S, d, N, K, W = 8, 16, 96, 3, 12
    scale = 1 / math.sqrt(d)
    Q, Kc, V = _rand((1, 2, N, d), 1000 + seed), _rand((1, 2, N, d), 1100 + seed), _rand((1, 2, N, d), 1200 + seed)
    LQ = _rand((1, 2, N // S, d), 1300 + seed)
    ksum, bsum = oracle.summarize(Kc, LQ, S, scale)
    idx, score, nsel = oracle.select(Q, ksum, bsum, S, K, scale)
    O, _ = oracle.attend(Q, Kc, V, idx, score, nsel, S, W, scale)
    for h in range(2):
        for i in (0, 7, 8, 9, 30, 63, 64, 95):
            w = oracle.brute_weights(Q, Kc, idx[0, h, i], score[0, h, i], nsel[0, h, i],
                                     0, h, i, i, S, W, scale)
            assert abs(w.sum() - 1.0) < 1e-12
            np.testing.assert_allclose(w @ V[0, h, :i + 1].numpy(), O[0, h, i], rtol=0, atol=1e-12)


def test_window_overlapping_a_selected_chunk_counts_twice(oracle):
    """A token inside both a selected chunk and the window enters through both terms."""
    S, d = 4, 8
    scale = 0.3
    Q, Kc, V = _rand((1, 1, 16, d), 1401), _rand((1, 1, 16, d), 1402), _rand((1, 1, 16, d), 1403)
    i = t = 13  # own chunk 3; chunk 2 = tokens 8..11 is eligible; window W = 4 -> 10..13
    idx = np.array([2], np.int32)
    s2 = 0.7
    w = oracle.brute_weights(Q, Kc, idx, np.array([s2]), 1, 0, 0, i, t, S, 4, scale)
    logits = (Kc[0, 0, :t + 1] @ Q[0, 0, i]).numpy() * scale
    zhat = math.exp(s2) + np.exp(logits[10:14]).sum()
    zc = np.exp(logits[8:12]).sum()
    want = np.zeros(t + 1)
    want[8:12] += np.exp(logits[8:12]) / zc * math.exp(s2) / zhat
    want[10:14] += np.exp(logits[10:14]) / zhat
    np.testing.assert_allclose(w, want, rtol=0, atol=1e-14)


def test_decode_form_equals_the_prefill_row(oracle):
    """The decode form (one query at an explicit position t, qpos) selects and attends
    exactly as row t of the prefill form over the same sequence: same kept chunks, same
    scores, same output and lse, and tokens after t (present in the keys and values)
    take no part."""
    g = np.random.default_rng(123)
    B, H, d, S, N, K, W, sc = 1, 2, 16, 64, 64 * 5 + 11, 3, 70, 0.3
    Q, Qcal, Kc, Vc = (torch.from_numpy(g.standard_normal((B, H, N, d))) for _ in range(4))
    LQ = torch.from_numpy(g.standard_normal((B, H, N // S, d)))
    ks, bs = oracle.summarize(Kc, LQ, S, sc)
    idx, score, nsel = oracle.select(Qcal, ks, bs, S, K, sc)
    O, lse = oracle.attend(Q, Kc, Vc, idx, score, nsel, S, W, sc)
    for t in (0, 63, 64, 130, 200, N - 1):
        qpos = np.full((B, 1), t, np.int32)
        i1, s1, n1 = oracle.select(Qcal[:, :, t:t + 1], ks, bs, S, K, sc, qpos=qpos)
        assert (n1 == nsel[:, :, t:t + 1]).all() and (i1 == idx[:, :, t:t + 1]).all(), t
        assert np.array_equal(s1, score[:, :, t:t + 1]), t
        Vj = Vc.clone()
        Vj[:, :, t + 1:] += 1000.0  # tokens after the query must not matter
        O1, l1 = oracle.attend(Q[:, :, t:t + 1], Kc, Vj, i1, s1, n1, S, W, sc, qpos=qpos)
        assert np.abs(O1[:, :, 0] - O[:, :, t]).max() < 1e-12, t
        assert np.abs(l1[:, :, 0] - lse[:, :, t]).max() < 1e-12, t
