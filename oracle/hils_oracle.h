/*
 * HiLS-Attention forward pass: float64 CPU oracle (declarations).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the bench's CPU
 * baseline leg may load this library. The CUDA library never includes this header,
 * and this oracle includes nothing from the CUDA library.
 *
 * Sources:
 *   [summary] "Hierarchical Sparse Attention Done Right: Toward Infinite Context
 *             Modeling", picx.dev summary page: Introduction (chunk mass and its two
 *             log-Z regimes), Methodology 1 (Eq. 7, Eq. 8), Methodology 2 (Eq. 10 and
 *             the definition of the surrogate chunk mass and its normaliser).
 *   [post]    the same title, rcap.io post: the per-query pseudocode figure
 *             (score every chunk, keep the top K, hierarchical combination, sliding
 *             window) and the deployment recipe (chunk 64, window 512, top-K 32).
 *
 * Layout conventions (shared by every function):
 *   A tensor is 4-D [B, H, T, D] with element (b, h, t, x) at
 *   ptr + b*sb + h*sh + t*st + x (strides in elements; the innermost stride is 1).
 *   A 3-D tensor [B, H, T] uses the same struct with x = 0.
 *   dtype: OR_F32 = float, OR_BF16 = raw bfloat16 bits (uint16), OR_F64 = double.
 *   Every stored element is widened exactly to double before any arithmetic.
 *   Outputs are plain contiguous row-major double/int arrays owned by the caller.
 *
 * Return value: 0 on success, -1 on an invalid argument.
 */
#ifndef HILS_ORACLE_H
#define HILS_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

typedef struct {
    const void *ptr;
    int dtype;
    long long sb, sh, st;
} or_tensor;

/* Threads used by every oracle call (OpenMP over independent (b, h, item) units). */
void or_set_threads(int n);
int or_get_threads(void);

/* Eq. 8: landmark softmax over each complete chunk, attention-weighted key k'_c and
 * entropy bias b'_c. G query heads share a key-value head (G = 1: one each).
 * K: [B,H/G,N,d]; LQ: [B,H,C,d] with C = N / S (floor); query head h reads key-value
 * head h / G. Ksum: [B,H,C,d] double; Bsum: [B,H,C] double. */
int or_summarize(int B, int H, int G, int d, int S, double scale,
                 or_tensor K, int N, or_tensor LQ,
                 double *Ksum, double *Bsum);

/* Eq. 7 with the calibrated query (Methodology 2): the surrogate log-mass of every
 * chunk for every query. Qcal: [B,H,Lq,d]; Ksum: [B,H,C,d]; Bsum: [B,H,C] (x = 0).
 * qpos: [B, Lq] query positions t, or NULL for t = i. A chunk c is eligible for the
 * query at t when c < min(floor(t / S), C), and, when excl_w = W > 0 (the window
 * exclusion), c * S < max(0, t - W + 1). out: [B,H,Lq,C]; ineligible = -inf. */
int or_score_all(int B, int H, int d, int S, int excl_w, double scale,
                 or_tensor Qcal, int Lq, const int *qpos,
                 or_tensor Ksum, or_tensor Bsum, int C, double *out);

/* Top-K over the eligible chunks of each group of G query heads, ranked by (the
 * group's largest score descending, chunk index ascending). The kept chunks are
 * listed in ascending chunk index. idx: [B,H/G,Lq,K] int (-1 padding), nsel:
 * [B,H/G,Lq] = min(K, number of eligible chunks); score: [B,H,Lq,K] double, each
 * head's own score of the kept chunks (-inf padding). */
int or_select(int B, int H, int G, int d, int S, int K, int excl_w, double scale,
              or_tensor Qcal, int Lq, const int *qpos,
              or_tensor Ksum, or_tensor Bsum, int C,
              int *idx, double *score, int *nsel);

/* Eq. 10: hierarchical softmax over the selected chunks (surrogate mass exp(score))
 * plus the sliding window [max(0, t-W+1), t] (exact token mass), with one joint
 * normaliser. Q: [B,H,Lq,d]; Kc, Vc: [B,H/G,L,d] (only positions <= t are read;
 * query head h reads key-value head h / G); idx: [B,H/G,Lq,K] int and nsel: [B,H/G,Lq]
 * (the group's kept chunks); score: [B,H,Lq,K] as an or_tensor with st = K (f32 or
 * f64). O: [B,H,Lq,d] double; lse: [B,H,Lq] double (may be NULL). */
int or_attend(int B, int H, int G, int d, int S, int K, int W, double scale,
              or_tensor Q, int Lq, const int *qpos,
              or_tensor Kc, or_tensor Vc,
              const int *idx, or_tensor score, const int *nsel,
              double *O, double *lse);

/* Token-level form of Eq. 10 for one query (b, h, i): writes w[j] for j in [0, t]
 * (t+1 entries). Used by tests to check sum_j w = 1 and o = w . V independently of
 * or_attend. */
int or_brute_weights(int H, int d, int S, int K, int W, double scale,
                     or_tensor Q, int b, int h, int i, int t,
                     or_tensor Kc, const int *idx_row, or_tensor score, long long score_off,
                     int nsel_row, double *w);

/* Exact chunk log-mass log Z_{i,c} = log sum_{j in chunk c} exp(scale * q_i . k_j)
 * (Introduction, chunk mass) for every selected chunk: out [B,H,Lq,K], -inf padding. */
int or_chunk_logmass(int B, int H, int d, int S, int K, double scale,
                     or_tensor Q, int Lq, or_tensor Kc,
                     const int *idx, const int *nsel, double *out);

#ifdef __cplusplus
}
#endif
#endif
