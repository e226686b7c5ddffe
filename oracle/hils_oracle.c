/*
 * HiLS-Attention forward pass: float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE. This is the slow, plainly written reference that the GPU
 * parity tests, the smoke check and the bench's CPU baseline compare against. Only
 * tests/, the smoke check and the bench's CPU baseline leg may load it; the CUDA
 * library neither links nor calls it, and it shares no code with that library.
 *
 * Every formula below is written from the pages, in their order and notation:
 *   [summary] "Hierarchical Sparse Attention Done Right: Toward Infinite Context
 *             Modeling", picx.dev summary page, Introduction (chunk mass Z_{i,c}),
 *             Methodology 1 (Eq. 7, Eq. 8) and Methodology 2 (Eq. 10; definition of
 *             s^_{i,c}, Z^_{i,c} and the normaliser Z^_i over the selected chunks and
 *             the sliding window).
 *   [post]    same title, rcap.io post, the per-query pseudocode figure (score every
 *             chunk, keep the top K, weight each chunk's own softmax output by its
 *             surrogate mass, add the sliding-window term).
 *
 * Readings of points the pages leave open (each is listed with its reason in the
 * design notes of the repository):
 *   - one scale 1/sqrt(d) (passed in as `scale`) multiplies every dot product; the
 *     entropy bias is added unscaled (Eq. 7).
 *   - chunk c is eligible for the query at position t when c < floor(t / S): only
 *     complete chunks strictly before the query's own chunk.
 *   - fewer than K eligible chunks: all of them are kept; the rest is padding.
 *   - the window is the W most recent tokens including the query's own, and it
 *     joins the selected chunks under one normaliser Z^_i; a token that is both in a
 *     selected chunk and in the window contributes through both terms.
 *   - top-K ties go to the lower chunk index; the kept list is reported in
 *     ascending chunk index.
 *   - a query with no selected chunk and an empty window gets o = 0, lse = -inf.
 *   - the window-exclusion variant (excl_w = W, the `flags` bit of the library): a
 *     chunk that lies wholly inside the query's window is not eligible, since the
 *     window already attends its tokens exactly; the chunk holding the window's first
 *     token, when the window starts inside a chunk, stays eligible (excluding it would
 *     leave its earlier tokens unreachable), so its window tokens still count twice.
 *   - grouped-query attention ([summary] Methodology 3, GQA adaptation): H query heads
 *     share H / G key-value heads, query head h reading key-value head h / G. Each query
 *     head has its own landmark queries, summaries and chunk scores; a group's G heads
 *     keep the same chunks, the top K of max over the group of s^_{h,i,c} (ties to the
 *     lower index); each head weights the kept chunks with its own s^_{h,i,c} in Eq. 10.
 *     G = 1 is plain multi-head attention.
 *
 * Arithmetic: every stored element is widened exactly to double. All sums run in
 * index order; the file must be compiled without floating-point contraction
 * (-ffp-contract=off) and without fast-math, so that a chunk score is the exact
 * sequence  acc = sum_x (q_x * k'_x)  (in x order), s = acc * scale + b'.
 */
#include "hils_oracle.h"

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int g_threads = 0;

void or_set_threads(int n) { g_threads = n > 0 ? n : 0; }

int or_get_threads(void) {
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- storage access */

static double widen(const or_tensor *x, long long off) {
    switch (x->dtype) {
    case OR_F32:
        return (double)((const float *)x->ptr)[off];
    case OR_BF16: {
        uint32_t bits = (uint32_t)((const uint16_t *)x->ptr)[off] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    default:
        return ((const double *)x->ptr)[off];
    }
}

static long long at(const or_tensor *x, int b, int h, long long t) {
    return (long long)b * x->sb + (long long)h * x->sh + t * x->st;
}

static void load_vec(const or_tensor *x, int b, int h, long long t, int d, double *out) {
    long long o = at(x, b, h, t);
    for (int j = 0; j < d; ++j) out[j] = widen(x, o + j);
}

static int valid_dtype(const or_tensor *x) {
    return x->ptr != NULL && (x->dtype == OR_F32 || x->dtype == OR_BF16 || x->dtype == OR_F64);
}

/* ------------------------------------------------------------------- arithmetic */

static double dot(const double *a, const double *b, int d) {
    double acc = 0.0;
    for (int j = 0; j < d; ++j) acc += a[j] * b[j];
    return acc;
}

/* Number of chunks the query at position t may select: complete chunks strictly
 * before its own chunk, capped by the number of summarised chunks. With the window
 * exclusion (excl_w = W > 0) only chunks that start before the window
 * [max(0, t-W+1), t], that is, that do not lie wholly inside it: c*S < max(0, t-W+1). */
static int eligible_chunks(int t, int S, int C, int excl_w) {
    int e = t >= 0 ? t / S : 0;
    if (e > C) e = C;
    if (excl_w > 0 && t >= 0) {
        const int w0 = t - excl_w + 1 > 0 ? t - excl_w + 1 : 0;
        const int nw = (w0 + S - 1) / S;
        if (e > nw) e = nw;
    }
    return e;
}

/* --------------------------------------------------------------- Eq. 8 summaries */

int or_summarize(int B, int H, int G, int d, int S, double scale,
                 or_tensor K, int N, or_tensor LQ,
                 double *Ksum, double *Bsum) {
    if (B < 0 || H < 0 || G <= 0 || H % G != 0 || d <= 0 || S <= 0 || N < 0) return -1;
    if (!valid_dtype(&K) || !valid_dtype(&LQ) || !Ksum || !Bsum) return -1;
    const int C = N / S;
    const long long units = (long long)B * H * C;
    if (units == 0) return 0;

#pragma omp parallel num_threads(or_get_threads())
    {
        double *lq = malloc(sizeof(double) * d);
        double *kj = malloc(sizeof(double) * d);
        double *logit = malloc(sizeof(double) * S);
#pragma omp for schedule(dynamic, 8)
        for (long long u = 0; u < units; ++u) {
            const int c = (int)(u % C);
            const int h = (int)((u / C) % H);
            const int b = (int)(u / ((long long)C * H));
            load_vec(&LQ, b, h, c, d, lq);

            /* landmark logits l_j = (q'_c . k_j) / sqrt(d) over the chunk's S keys (of the
               query head's key-value head h / G) */
            double m = -INFINITY;
            for (int j = 0; j < S; ++j) {
                load_vec(&K, b, h / G, (long long)c * S + j, d, kj);
                logit[j] = dot(lq, kj, d) * scale;
                if (logit[j] > m) m = logit[j];
            }
            /* p = softmax(l) */
            double z = 0.0;
            for (int j = 0; j < S; ++j) z += exp(logit[j] - m);

            /* k'_c = sum_j p_j k_j ;  b'_c = -sum_j p_j log p_j  (0 log 0 = 0) */
            double *ks = Ksum + u * d;
            for (int x = 0; x < d; ++x) ks[x] = 0.0;
            double entropy = 0.0;
            for (int j = 0; j < S; ++j) {
                const double p = exp(logit[j] - m) / z;
                load_vec(&K, b, h / G, (long long)c * S + j, d, kj);
                for (int x = 0; x < d; ++x) ks[x] += p * kj[x];
                if (p > 0.0) entropy -= p * log(p);
            }
            Bsum[u] = entropy;
        }
        free(lq);
        free(kj);
        free(logit);
    }
    return 0;
}

/* ------------------------------------------------------- Eq. 7 chunk scores + top-K */

/* s^_{i,c} = (q~_i . k'_c) / sqrt(d) + b'_c, in the fixed order stated above. */
static double chunk_score(const double *q, const or_tensor *Ksum, const or_tensor *Bsum,
                          int b, int h, int c, int d, double scale, double *kbuf) {
    load_vec(Ksum, b, h, c, d, kbuf);
    const double acc = dot(q, kbuf, d);
    const double bias = widen(Bsum, at(Bsum, b, h, c));
    return acc * scale + bias;
}

int or_score_all(int B, int H, int d, int S, int excl_w, double scale,
                 or_tensor Qcal, int Lq, const int *qpos,
                 or_tensor Ksum, or_tensor Bsum, int C, double *out) {
    if (B < 0 || H < 0 || d <= 0 || S <= 0 || Lq < 0 || C < 0 || excl_w < 0 || !out) return -1;
    if (!valid_dtype(&Qcal) || (C > 0 && (!valid_dtype(&Ksum) || !valid_dtype(&Bsum)))) return -1;
    const long long units = (long long)B * H * Lq;
#pragma omp parallel num_threads(or_get_threads())
    {
        double *q = malloc(sizeof(double) * d);
        double *kb = malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 4)
        for (long long u = 0; u < units; ++u) {
            const int i = (int)(u % Lq);
            const int h = (int)((u / Lq) % H);
            const int b = (int)(u / ((long long)Lq * H));
            const int t = qpos ? qpos[(long long)b * Lq + i] : i;
            const int ne = eligible_chunks(t, S, C, excl_w);
            load_vec(&Qcal, b, h, i, d, q);
            double *row = out + u * C;
            for (int c = 0; c < C; ++c)
                row[c] = c < ne ? chunk_score(q, &Ksum, &Bsum, b, h, c, d, scale, kb) : -INFINITY;
        }
        free(q);
        free(kb);
    }
    return 0;
}

typedef struct {
    double s;
    int c;
} scored;

/* ranking order: higher score first, lower chunk index on equal scores */
static int by_rank(const void *pa, const void *pb) {
    const scored *a = pa, *b = pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->c > b->c) - (a->c < b->c);
}

static int by_index(const void *pa, const void *pb) {
    const scored *a = pa, *b = pb;
    return (a->c > b->c) - (a->c < b->c);
}

int or_select(int B, int H, int G, int d, int S, int K, int excl_w, double scale,
              or_tensor Qcal, int Lq, const int *qpos,
              or_tensor Ksum, or_tensor Bsum, int C,
              int *idx, double *score, int *nsel) {
    if (B < 0 || H < 0 || G <= 0 || H % G != 0 || d <= 0 || S <= 0 || K < 0 || Lq < 0 || C < 0 || excl_w < 0) return -1;
    if (!valid_dtype(&Qcal) || !idx || !score || !nsel) return -1;
    if (C > 0 && (!valid_dtype(&Ksum) || !valid_dtype(&Bsum))) return -1;
    const int Hk = H / G;
    const long long units = (long long)B * Hk * Lq;  /* one per (b, group, query) */
#pragma omp parallel num_threads(or_get_threads())
    {
        double *q = malloc(sizeof(double) * d * G);
        double *kb = malloc(sizeof(double) * d);
        scored *all = malloc(sizeof(scored) * (C > 0 ? C : 1));
#pragma omp for schedule(dynamic, 4)
        for (long long u = 0; u < units; ++u) {
            const int i = (int)(u % Lq);
            const int g = (int)((u / Lq) % Hk);
            const int b = (int)(u / ((long long)Lq * Hk));
            const int t = qpos ? qpos[(long long)b * Lq + i] : i;
            const int ne = eligible_chunks(t, S, C, excl_w);
            for (int hh = 0; hh < G; ++hh) load_vec(&Qcal, b, g * G + hh, i, d, q + (long long)hh * d);
            /* the group's selection score of chunk c: the largest of its heads' s^ */
            for (int c = 0; c < ne; ++c) {
                double m = -INFINITY;
                for (int hh = 0; hh < G; ++hh) {
                    const double sc = chunk_score(q + (long long)hh * d, &Ksum, &Bsum, b, g * G + hh, c, d, scale, kb);
                    if (sc > m) m = sc;
                }
                all[c].s = m;
                all[c].c = c;
            }
            qsort(all, ne, sizeof(scored), by_rank);
            const int n = ne < K ? ne : K;
            qsort(all, n, sizeof(scored), by_index);
            for (int r = 0; r < K; ++r) idx[u * K + r] = r < n ? all[r].c : -1;
            nsel[u] = n;
            /* each head's own s^ of the kept chunks */
            for (int hh = 0; hh < G; ++hh) {
                const long long uh = ((long long)b * H + g * G + hh) * Lq + i;
                for (int r = 0; r < K; ++r)
                    score[uh * K + r] = r < n ? chunk_score(q + (long long)hh * d, &Ksum, &Bsum, b, g * G + hh,
                                                            all[r].c, d, scale, kb)
                                              : -INFINITY;
            }
        }
        free(q);
        free(kb);
        free(all);
    }
    return 0;
}

/* ------------------------------------------------ Eq. 10 hierarchical combination */

/* Softmax-weighted value of one chunk for query q: sum_{j in T_c} e^{l_j}/Z_c v_j. */
static void chunk_attention(const double *q, const or_tensor *Kc, const or_tensor *Vc,
                            int b, int h, int c, int S, int d, double scale,
                            double *logit, double *kv, double *out) {
    double m = -INFINITY;
    for (int j = 0; j < S; ++j) {
        load_vec(Kc, b, h, (long long)c * S + j, d, kv);
        logit[j] = dot(q, kv, d) * scale;
        if (logit[j] > m) m = logit[j];
    }
    double z = 0.0;
    for (int j = 0; j < S; ++j) z += exp(logit[j] - m);
    for (int x = 0; x < d; ++x) out[x] = 0.0;
    for (int j = 0; j < S; ++j) {
        const double w = exp(logit[j] - m) / z;
        load_vec(Vc, b, h, (long long)c * S + j, d, kv);
        for (int x = 0; x < d; ++x) out[x] += w * kv[x];
    }
}

int or_attend(int B, int H, int G, int d, int S, int K, int W, double scale,
              or_tensor Q, int Lq, const int *qpos,
              or_tensor Kc, or_tensor Vc,
              const int *idx, or_tensor score, const int *nsel,
              double *O, double *lse) {
    if (B < 0 || H < 0 || G <= 0 || H % G != 0 || d <= 0 || S <= 0 || K < 0 || W < 0 || Lq < 0) return -1;
    if (!valid_dtype(&Q) || !valid_dtype(&Kc) || !valid_dtype(&Vc) || !O) return -1;
    if (K > 0 && (!idx || !nsel || !valid_dtype(&score))) return -1;
    const long long units = (long long)B * H * Lq;
#pragma omp parallel num_threads(or_get_threads())
    {
        double *q = malloc(sizeof(double) * d);
        double *kv = malloc(sizeof(double) * d);
        double *logit = malloc(sizeof(double) * S);
        double *vecs = malloc(sizeof(double) * d * (K > 0 ? K : 1));
        double *mass = malloc(sizeof(double) * (K > 0 ? K : 1));
        double *wlogit = malloc(sizeof(double) * (W > 0 ? W : 1));
#pragma omp for schedule(dynamic, 4)
        for (long long u = 0; u < units; ++u) {
            const int i = (int)(u % Lq);
            const int h = (int)((u / Lq) % H);
            const int b = (int)(u / ((long long)Lq * H));
            const int t = qpos ? qpos[(long long)b * Lq + i] : i;
            const int hk = h / G;                              /* key-value head */
            const long long ug = ((long long)b * (H / G) + hk) * Lq + i;  /* the group's kept list */
            load_vec(&Q, b, h, i, d, q);

            /* selected chunks: log surrogate mass s^_{i,c} and chunk-local output */
            int nc = 0;
            const int ns = K > 0 ? nsel[ug] : 0;
            for (int r = 0; r < ns && r < K; ++r) {
                const int c = idx[ug * K + r];
                if (c < 0) continue;
                mass[nc] = widen(&score, at(&score, b, h, i) + r);
                chunk_attention(q, &Kc, &Vc, b, hk, c, S, d, scale, logit, kv, vecs + (long long)nc * d);
                ++nc;
            }
            /* window tokens [max(0, t-W+1), t]: exact token logits */
            const int w0 = t - W + 1 > 0 ? t - W + 1 : 0;
            const int nw = W > 0 ? t - w0 + 1 : 0;
            for (int j = 0; j < nw; ++j) {
                load_vec(&Kc, b, hk, w0 + j, d, kv);
                wlogit[j] = dot(q, kv, d) * scale;
            }

            /* Z^_i = sum_c e^{s^_c} + sum_{j in window} e^{l_ij}, shifted by the max */
            double M = -INFINITY;
            for (int r = 0; r < nc; ++r) if (mass[r] > M) M = mass[r];
            for (int j = 0; j < nw; ++j) if (wlogit[j] > M) M = wlogit[j];
            double *o = O + u * d;
            for (int x = 0; x < d; ++x) o[x] = 0.0;
            if (nc + nw == 0 || M == -INFINITY) {
                if (lse) lse[u] = -INFINITY;
                continue;
            }
            double zhat = 0.0;
            for (int r = 0; r < nc; ++r) {
                const double e = exp(mass[r] - M);
                zhat += e;
                for (int x = 0; x < d; ++x) o[x] += e * vecs[(long long)r * d + x];
            }
            for (int j = 0; j < nw; ++j) {
                const double e = exp(wlogit[j] - M);
                zhat += e;
                load_vec(&Vc, b, hk, w0 + j, d, kv);
                for (int x = 0; x < d; ++x) o[x] += e * kv[x];
            }
            for (int x = 0; x < d; ++x) o[x] /= zhat;
            if (lse) lse[u] = M + log(zhat);
        }
        free(q);
        free(kv);
        free(logit);
        free(vecs);
        free(mass);
        free(wlogit);
    }
    return 0;
}

int or_brute_weights(int H, int d, int S, int K, int W, double scale,
                     or_tensor Q, int b, int h, int i, int t,
                     or_tensor Kc, const int *idx_row, or_tensor score, long long score_off,
                     int nsel_row, double *w) {
    (void)H;
    if (d <= 0 || S <= 0 || K < 0 || W < 0 || t < 0 || !w) return -1;
    if (!valid_dtype(&Q) || !valid_dtype(&Kc)) return -1;
    double *q = malloc(sizeof(double) * d);
    double *kv = malloc(sizeof(double) * d);
    double *s = malloc(sizeof(double) * (t + 1));
    int rc = 0;
    load_vec(&Q, b, h, i, d, q);
    /* token logits s_ij for every j <= t */
    for (int j = 0; j <= t; ++j) {
        load_vec(&Kc, b, h, j, d, kv);
        s[j] = dot(q, kv, d) * scale;
    }
    const int w0 = t - W + 1 > 0 ? t - W + 1 : 0;
    /* max over every log-mass that enters Z^_i */
    double M = -INFINITY;
    for (int r = 0; r < nsel_row && r < K; ++r) {
        if (idx_row[r] < 0) continue;
        if ((long long)(idx_row[r] + 1) * S - 1 > t) { rc = -1; goto done; }
        const double sh = widen(&score, score_off + r);
        if (sh > M) M = sh;
    }
    if (W > 0)
        for (int j = w0; j <= t; ++j) if (s[j] > M) M = s[j];
    for (int j = 0; j <= t; ++j) w[j] = 0.0;
    if (M == -INFINITY) goto done;

    double zhat = 0.0;
    for (int r = 0; r < nsel_row && r < K; ++r)
        if (idx_row[r] >= 0) zhat += exp(widen(&score, score_off + r) - M);
    if (W > 0)
        for (int j = w0; j <= t; ++j) zhat += exp(s[j] - M);

    /* chunk term: w_ij = e^{s_ij} / Z_{i,c(j)} * Z^_{i,c(j)} / Z^_i */
    for (int r = 0; r < nsel_row && r < K; ++r) {
        const int c = idx_row[r];
        if (c < 0) continue;
        double mc = -INFINITY, zc = 0.0;
        for (int j = c * S; j < (c + 1) * S; ++j) if (s[j] > mc) mc = s[j];
        for (int j = c * S; j < (c + 1) * S; ++j) zc += exp(s[j] - mc);
        const double inter = exp(widen(&score, score_off + r) - M) / zhat;
        for (int j = c * S; j < (c + 1) * S; ++j) w[j] += exp(s[j] - mc) / zc * inter;
    }
    /* window term: e^{s_ij} / Z^_i */
    if (W > 0)
        for (int j = w0; j <= t; ++j) w[j] += exp(s[j] - M) / zhat;
done:
    free(q);
    free(kv);
    free(s);
    return rc;
}

/* ----------------------------------------------------- exact chunk mass (Introduction) */

int or_chunk_logmass(int B, int H, int d, int S, int K, double scale,
                     or_tensor Q, int Lq, or_tensor Kc,
                     const int *idx, const int *nsel, double *out) {
    if (B < 0 || H < 0 || d <= 0 || S <= 0 || K < 0 || Lq < 0 || !out) return -1;
    if (!valid_dtype(&Q) || !valid_dtype(&Kc) || (K > 0 && (!idx || !nsel))) return -1;
    const long long units = (long long)B * H * Lq;
#pragma omp parallel num_threads(or_get_threads())
    {
        double *q = malloc(sizeof(double) * d);
        double *kv = malloc(sizeof(double) * d);
        double *logit = malloc(sizeof(double) * S);
#pragma omp for schedule(dynamic, 4)
        for (long long u = 0; u < units; ++u) {
            const int i = (int)(u % Lq);
            const int h = (int)((u / Lq) % H);
            const int b = (int)(u / ((long long)Lq * H));
            load_vec(&Q, b, h, i, d, q);
            for (int r = 0; r < K; ++r) {
                const int c = idx[u * K + r];
                if (r >= nsel[u] || c < 0) {
                    out[u * K + r] = -INFINITY;
                    continue;
                }
                double m = -INFINITY;
                for (int j = 0; j < S; ++j) {
                    load_vec(&Kc, b, h, (long long)c * S + j, d, kv);
                    logit[j] = dot(q, kv, d) * scale;
                    if (logit[j] > m) m = logit[j];
                }
                double z = 0.0;
                for (int j = 0; j < S; ++j) z += exp(logit[j] - m);
                out[u * K + r] = m + log(z);
            }
        }
        free(q);
        free(kv);
        free(logit);
    }
    return 0;
}
