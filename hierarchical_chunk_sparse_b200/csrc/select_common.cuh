// Exact top-K building blocks shared by the select kernels: "Hierarchical Sparse
// Attention Done Right" (picx.dev summary), Eq. 7 and Methodology 2, and the rcap.io
// post's pseudocode figure (keep the top K chunks per query).
//
// Exactness rests on interval screening. Each chunk carries a float32 screen value s
// with a rigorous radius e; certainly-in and certainly-out chunks are settled by the
// intervals alone, and only the chunks in between get the float64 score
//   x_c = (sum_x q~_x k'_x) * scale + b'_c   (every product and sum rounded to float64,
//                                             in x order).
// The warp routines below keep a running exact top-K list over 128-chunk tiles, one
// lane per chunk.
#pragma once
#include <float.h>
#include <limits.h>
#include <math.h>

#include <type_traits>

#include "hils_internal.cuh"

namespace hils {
namespace {

constexpr int kWarpKernelWarps = 8;  // warps (queries) per CTA of the warp-per-query select
constexpr int kWarpKernelThreads = kWarpKernelWarps * 32;
constexpr int kTile = 128;      // chunks scored per warp step
constexpr int kMaxK = 32;
constexpr int kListBytes = 768; // one list of <= 32 entries in the workspace

// One list of kept entries (in shared memory or the workspace).
struct EntryList {
    double x[kMaxK];   // exact score, NaN if not computed
    int idx[kMaxK];
    float s[kMaxK];
    float e[kMaxK];
    int n;
    float bound;       // lower bound on the K-th largest lo of the range the list covers
};
static_assert(sizeof(EntryList) <= kListBytes, "list size");

template <int R>
struct Slots {
    int idx[R];
    float s[R];
    float e[R];
    double x[R];
};

struct QueryCtx {
    const void *qrow;       // q~_i in global memory (for exact scores)
    const void *khead;      // k'_0 of this (b, h)
    int64_t kst;
    const float *bhead;     // b'_0 of this (b, h)
    float scale;
};

template <typename T, int D>
__device__ double exact_score(const QueryCtx &q, int c) {
    // rows are read with 16-byte loads, half a row at a time, before the fixed-order
    // float64 chain runs over them
    constexpr int kN = Vec<T>::kN, kHalf = D / kN / 2;
    const uint4 *qr = static_cast<const uint4 *>(q.qrow);
    const uint4 *kr = reinterpret_cast<const uint4 *>(static_cast<const T *>(q.khead) + (int64_t)c * q.kst);
    double acc = 0.0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint4 qv[kHalf], kv[kHalf];
#pragma unroll
        for (int u = 0; u < kHalf; ++u) {
            qv[u] = __ldg(qr + h * kHalf + u);
            kv[u] = __ldg(kr + h * kHalf + u);
        }
#pragma unroll
        for (int u = 0; u < kHalf; ++u) {
            float qf[kN], kf[kN];
            widen(qv[u], qf, T());
            widen(kv[u], kf, T());
#pragma unroll
            for (int i = 0; i < kN; ++i) acc = __dadd_rn(acc, __dmul_rn((double)qf[i], (double)kf[i]));
        }
    }
    return __dadd_rn(__dmul_rn(acc, (double)q.scale), (double)q.bhead[c]);
}

// Float32 screen value and its error radius for chunk c; qs = query in shared memory.
template <typename T, int D>
__device__ __forceinline__ void screen(const QueryCtx &q, const float *qs, int c, float &s, float &e) {
    const uint4 *kr = reinterpret_cast<const uint4 *>(static_cast<const T *>(q.khead) + (int64_t)c * q.kst);
    constexpr int kN = Vec<T>::kN;
    float dot = 0.f, ad = 0.f;
#pragma unroll
    for (int u = 0; u < D / kN; ++u) {
        float kf[kN];
        widen(__ldg(kr + u), kf, T());
#pragma unroll
        for (int i = 0; i < kN; ++i) {
            const float qv = qs[u * kN + i];
            dot = fmaf(qv, kf[i], dot);
            ad = fmaf(fabsf(qv), fabsf(kf[i]), ad);
        }
    }
    s = fmaf(dot, q.scale, q.bhead[c]);
    e = fmaf(q.scale * ad, (float)(D + 2) * 0x1p-23f, fabsf(s) * 0x1p-22f);
}

// Exact top-K of the warp's pool (R slots per lane, idx < 0 = empty). Returns the
// lane's mask of kept slots. Uniform control flow across the warp.
// `bound` receives a lower bound on the pool's K-th largest lo (s_K - e_max, rounded
// down), or -inf when the pool holds at most K entries. Any chunk whose hi lies below
// the bound of some subset of its competitors is certainly out.
template <typename T, int D, int R, typename Ctx>
__device__ unsigned warp_topk(Slots<R> &p, int K, const Ctx &q, float &bound) {
    const int lane = threadIdx.x & 31;
    unsigned valid = 0;
#pragma unroll
    for (int r = 0; r < R; ++r)
        if (p.idx[r] >= 0) valid |= 1u << r;
    const int n = __reduce_add_sync(kFull, __popc(valid));
    bound = -INFINITY;
    if (n <= K) return valid;

    float em = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r)
        if (valid >> r & 1) em = fmaxf(em, p.e[r]);
    em = warp_max(em);

    // K-th and (K+1)-th largest screen values (duplicates counted separately)
    unsigned taken = 0;
    float sK = 0.f, sK1 = 0.f;
    for (int it = 0; it <= K; ++it) {
        unsigned best = 0u;
        int bslot = -1;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            if ((valid & ~taken) >> r & 1) {
                const unsigned k = ordered_key(p.s[r]);
                if (k > best) {
                    best = k;
                    bslot = r;
                }
            }
        }
        const unsigned wmax = __reduce_max_sync(kFull, best);
        const unsigned owners = __ballot_sync(kFull, bslot >= 0 && best == wmax);
        if (lane == __ffs(owners) - 1) taken |= 1u << bslot;
        const float v = key_to_float(wmax);
        if (it == K - 1) sK = v;
        sK1 = v;
    }
    const float lo_cut = __fsub_rd(sK, em);
    const float hi_cut = __fadd_ru(sK1, em);
    bound = lo_cut;

    unsigned in = 0, band = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (valid >> r & 1) {
            const float lo = __fsub_rd(p.s[r], p.e[r]);
            const float hi = __fadd_ru(p.s[r], p.e[r]);
            if (lo > hi_cut) in |= 1u << r;
            else if (hi >= lo_cut) band |= 1u << r;
        }
    }
    const int need = K - __reduce_add_sync(kFull, __popc(in));
    if (need > 0) {
#pragma unroll
        for (int r = 0; r < R; ++r)
            if ((band >> r & 1) && isnan(p.x[r])) p.x[r] = exact_score<T, D>(q, p.idx[r]);
        unsigned chosen = 0;
        for (int it = 0; it < need; ++it) {
            double bx = -INFINITY;
            int bi = INT_MAX;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if ((band & ~chosen) >> r & 1) {
                    if (p.x[r] > bx || (p.x[r] == bx && p.idx[r] < bi)) {
                        bx = p.x[r];
                        bi = p.idx[r];
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ox = __shfl_xor_sync(kFull, bx, o);
                const int oi = __shfl_xor_sync(kFull, bi, o);
                if (ox > bx || (ox == bx && oi < bi)) {
                    bx = ox;
                    bi = oi;
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r)
                if (((band & ~chosen) >> r & 1) && p.idx[r] == bi) chosen |= 1u << r;
        }
        in |= chosen;
    }
    return in;
}

// Appends the lane's kept slots to `list` after its first `base` entries; returns the
// new length.
template <int R>
__device__ int warp_append(const Slots<R> &p, unsigned keep, EntryList &list, int base) {
    const int lane = threadIdx.x & 31;
    const int cnt = __popc(keep);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
    }
    int pos = base + incl - cnt;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (keep >> r & 1) {
            list.idx[pos] = p.idx[r];
            list.s[pos] = p.s[r];
            list.e[pos] = p.e[r];
            list.x[pos] = p.x[r];
            ++pos;
        }
    }
    return base + __shfl_sync(kFull, incl, 31);
}

// Scores chunks [c0, c1) in tiles of 128 and leaves their exact top-K in `list`.
template <typename T, int D, typename Ctx>
__device__ void warp_scan(const Ctx &q, const float *qs, int c0, int c1, int K, EntryList &list) {
    const int lane = threadIdx.x & 31;
    int n = 0;
    for (int base = c0; base < c1; base += kTile) {
        Slots<5> p;
        // slot 0 carries the running list, one entry per lane
        p.idx[0] = lane < n ? list.idx[lane] : -1;
        p.s[0] = lane < n ? list.s[lane] : 0.f;
        p.e[0] = lane < n ? list.e[lane] : 0.f;
        p.x[0] = lane < n ? list.x[lane] : 0.0;
#pragma unroll
        for (int r = 1; r < 5; ++r) {
            const int c = base + lane + 32 * (r - 1);
            p.idx[r] = c < c1 ? c : -1;
            p.s[r] = 0.f;
            p.e[r] = 0.f;
            p.x[r] = __longlong_as_double(0x7ff8000000000000ll);  // NaN: not computed
            if (c < c1) screen<T, D>(q, qs, c, p.s[r], p.e[r]);
        }
        float bnd;
        const unsigned keep = warp_topk<T, D, 5>(p, K, q, bnd);
        __syncwarp();
        n = warp_append<5>(p, keep, list, 0);
        __syncwarp();
    }
    if (lane == 0) list.n = n;
    __syncwarp();
}

// Reduces `nlists` lists (<= R*32 entries in total) to their exact top-K in `out`.
template <typename T, int D, int R, typename Ctx>
__device__ void warp_merge(const Ctx &q, const EntryList *lists, int nlists, bool from_global, int K,
                           EntryList &out) {
    const int lane = threadIdx.x & 31;
    Slots<R> p;
#pragma unroll
    for (int r = 0; r < R; ++r) p.idx[r] = -1;
    // entry (l, j) -> pool position l*K + j -> slot (pos / 32) of lane (pos % 32)
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int pos = r * 32 + lane;
        const int l = pos / (K > 0 ? K : 1), j = pos - l * (K > 0 ? K : 1);
        if (K > 0 && l < nlists) {
            const EntryList &L = lists[l];
            const int ln = from_global ? __ldcg(&L.n) : L.n;
            if (j < ln) {
                p.idx[r] = from_global ? __ldcg(&L.idx[j]) : L.idx[j];
                p.s[r] = from_global ? __ldcg(&L.s[j]) : L.s[j];
                p.e[r] = from_global ? __ldcg(&L.e[j]) : L.e[j];
                p.x[r] = from_global ? __ldcg(&L.x[j]) : L.x[j];
            }
        }
    }
    float bnd;
    const unsigned keep = warp_topk<T, D, R>(p, K, q, bnd);
    __syncwarp();
    const int n = warp_append<R>(p, keep, out, 0);
    if (lane == 0) out.n = n;
    __syncwarp();
}

// Writes a kept list in ascending chunk index, padded to K.
__device__ void warp_write(const EntryList &list, int K, int64_t qi, int32_t *idx, float *score, int32_t *nsel) {
    const int lane = threadIdx.x & 31;
    const int n = list.n;
    if (lane < n) {
        const int me = list.idx[lane];
        int rank = 0;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) rank += (j < n && list.idx[j] < me) ? 1 : 0;
        idx[qi * K + rank] = me;
        score[qi * K + rank] = list.s[lane];
    } else if (lane < K) {
        idx[qi * K + lane] = -1;
        score[qi * K + lane] = -INFINITY;
    }
    if (lane == 0) nsel[qi] = n;
}

template <typename T, int D>
__device__ __forceinline__ QueryCtx make_ctx(const SelectArgs &a, int64_t qi, int &t) {
    const int q32 = (int)qi;  // query counts are checked to fit in int
    const int i = q32 % a.Lq;
    const int bh = q32 / a.Lq;
    const int h = bh % a.H;
    const int b = bh / a.H;
    t = a.qpos ? a.qpos[(int64_t)b * a.Lq + i] + a.qpos_bias : i;
    QueryCtx q;
    q.qrow = static_cast<const T *>(a.Qcal.ptr) + b * a.Qcal.sb + h * a.Qcal.sh + i * a.Qcal.st;
    q.khead = static_cast<const T *>(a.Ksum.ptr) + b * a.Ksum.sb + h * a.Ksum.sh;
    q.kst = a.Ksum.st;
    q.bhead = a.Bsum + ((int64_t)b * a.H + h) * a.C;
    q.scale = a.scale;
    return q;
}

// Chunks the query at position t may select: complete chunks before its own chunk,
// capped by C; with the window exclusion (excl_w = W > 0) only those that start before
// the window's first token max(0, t - W + 1), i.e. that do not lie wholly inside it.
__device__ __forceinline__ int eligible(int t, int C, int excl_w) {
    int e = t >= 0 ? t / kChunk : 0;
    e = e < C ? e : C;
    if (excl_w > 0 && t >= 0) {
        const int w0 = t - excl_w + 1 > 0 ? t - excl_w + 1 : 0;
        const int nw = (w0 + kChunk - 1) / kChunk;
        e = e < nw ? e : nw;
    }
    return e;
}

template <typename T, int D>
__device__ void load_query_f32(const QueryCtx &q, float *qs) {
    const T *qr = static_cast<const T *>(q.qrow);
    for (int x = threadIdx.x & 31; x < D; x += 32) qs[x] = (float)qr[x];
}

// ---- grouped-query selection ("Hierarchical Sparse Attention Done Right", summary page,
// Methodology 3, GQA adaptation): the G heads of a group keep the chunks with the largest
// maximum over the group of s^_{h,i,c}. A group chunk's interval is [max lo_h, max hi_h]
// over its heads' intervals, which contains the maximum of the heads' float64 scores; its
// float64 value is that maximum.
constexpr int kMaxGroup = kMaxGroupHeads;

struct GroupCtx {
    QueryCtx head;          // the group's first query head
    int64_t qsh, ksh, bsh;  // head strides of Q~, of k' (elements) and of b' (floats)
    int G;
};

__device__ __forceinline__ QueryCtx head_ctx(const GroupCtx &g, int hh, int es) {
    QueryCtx q = g.head;
    q.qrow = static_cast<const uint8_t *>(g.head.qrow) + (int64_t)hh * g.qsh * es;
    q.khead = static_cast<const uint8_t *>(g.head.khead) + (int64_t)hh * g.ksh * es;
    q.bhead = g.head.bhead + (int64_t)hh * g.bsh;
    return q;
}

// A centre and radius whose interval [s - e, s + e] contains [lo, hi] (finite): the
// midpoint's rounding is within 2^-24 |s|.
__device__ __forceinline__ void interval_mid(float lo, float hi, float &s, float &e) {
    s = 0.5f * lo + 0.5f * hi;
    e = __fadd_ru(__fmul_ru(__fsub_ru(hi, lo), 0.5f), fabsf(s) * 0x1p-23f);
}

// Folds one head's interval s +- e into the group's running [lo, hi].
__device__ __forceinline__ void fold_interval(float s, float e, float &lo, float &hi) {
    lo = fmaxf(lo, __fsub_rd(s, e));
    hi = fmaxf(hi, __fadd_ru(s, e));
}

template <typename T, int D>
__device__ __forceinline__ void screen(const GroupCtx &g, const float *qs, int c, float &s, float &e) {
    float lo = -INFINITY, hi = -INFINITY;
    for (int hh = 0; hh < g.G; ++hh) {
        float sh, eh;
        screen<T, D>(head_ctx(g, hh, (int)sizeof(T)), qs + hh * D, c, sh, eh);
        fold_interval(sh, eh, lo, hi);
    }
    interval_mid(lo, hi, s, e);
}

// The largest of the heads' float64 scores; two heads' fixed-order chains run side by
// side (each in its own x order, as for one head), rows read a quarter at a time.
template <typename T, int D>
__device__ double exact_score(const GroupCtx &g, int c) {
    constexpr int kN = Vec<T>::kN, kQ = D / kN / 4;
    double m = -INFINITY;
    for (int h0 = 0; h0 < g.G; h0 += 2) {
        const bool two = h0 + 1 < g.G;
        const QueryCtx q0 = head_ctx(g, h0, (int)sizeof(T));
        const QueryCtx q1 = head_ctx(g, two ? h0 + 1 : h0, (int)sizeof(T));
        const uint4 *qr[2] = {static_cast<const uint4 *>(q0.qrow), static_cast<const uint4 *>(q1.qrow)};
        const uint4 *kr[2] = {reinterpret_cast<const uint4 *>(static_cast<const T *>(q0.khead) + (int64_t)c * q0.kst),
                              reinterpret_cast<const uint4 *>(static_cast<const T *>(q1.khead) + (int64_t)c * q1.kst)};
        double acc[2] = {0.0, 0.0};
#pragma unroll
        for (int part = 0; part < 4; ++part) {
            uint4 qv[2][kQ], kv[2][kQ];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int u = 0; u < kQ; ++u) {
                    qv[j][u] = __ldg(qr[j] + part * kQ + u);
                    kv[j][u] = __ldg(kr[j] + part * kQ + u);
                }
#pragma unroll
            for (int u = 0; u < kQ; ++u) {
                float qf[2][kN], kf[2][kN];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    widen(qv[j][u], qf[j], T());
                    widen(kv[j][u], kf[j], T());
                }
#pragma unroll
                for (int i = 0; i < kN; ++i)
#pragma unroll
                    for (int j = 0; j < 2; ++j) acc[j] = __dadd_rn(acc[j], __dmul_rn((double)qf[j][i], (double)kf[j][i]));
            }
        }
        m = fmax(m, __dadd_rn(__dmul_rn(acc[0], (double)q0.scale), (double)q0.bhead[c]));
        if (two) m = fmax(m, __dadd_rn(__dmul_rn(acc[1], (double)q1.scale), (double)q1.bhead[c]));
    }
    return m;
}

// qg = (b, group, i): the group's first head, its strides, and the query's position
template <typename T, int D>
__device__ __forceinline__ GroupCtx make_group_ctx(const SelectArgs &a, int64_t qg, int &t, int &b, int &g, int &i) {
    const int Hk = a.H / a.G;
    const int q32 = (int)qg;
    i = q32 % a.Lq;
    const int bg = q32 / a.Lq;
    g = bg % Hk;
    b = bg / Hk;
    t = a.qpos ? a.qpos[(int64_t)b * a.Lq + i] + a.qpos_bias : i;
    const int h0 = g * a.G;
    GroupCtx q;
    q.head.qrow = static_cast<const T *>(a.Qcal.ptr) + b * a.Qcal.sb + h0 * a.Qcal.sh + i * a.Qcal.st;
    q.head.khead = static_cast<const T *>(a.Ksum.ptr) + b * a.Ksum.sb + h0 * a.Ksum.sh;
    q.head.kst = a.Ksum.st;
    q.head.bhead = a.Bsum + ((int64_t)b * a.H + h0) * a.C;
    q.head.scale = a.scale;
    q.qsh = a.Qcal.sh;
    q.ksh = a.Ksum.sh;
    q.bsh = a.C;
    q.G = a.G;
    return q;
}

// Writes a group's kept list (ascending chunk index, padded to K) for the group, and each
// head's own float32 screen value of the kept chunks.
template <typename T, int D>
__device__ void group_write(const GroupCtx &q, const float *qs, const EntryList &list, const SelectArgs &a,
                            int64_t qg, int b, int g, int i) {
    const int lane = threadIdx.x & 31;
    const int K = a.topk, n = list.n;
    int rank = lane, me = -1;
    if (lane < n) {
        me = list.idx[lane];
        rank = 0;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) rank += (j < n && list.idx[j] < me) ? 1 : 0;
    }
    if (lane < K) a.idx[qg * K + rank] = lane < n ? me : -1;
    for (int hh = 0; hh < q.G; ++hh) {
        const int64_t qh = ((int64_t)b * a.H + g * a.G + hh) * a.Lq + i;
        float sh = -INFINITY, eh;
        if (lane < n) screen<T, D>(head_ctx(q, hh, (int)sizeof(T)), qs + hh * D, me, sh, eh);
        if (lane < K) a.score[qh * K + rank] = sh;
    }
    if (lane == 0) a.nsel[qg] = n;
}

// Upper-tail standard normal quantile z with P(Z > z) = p, 0 < p <= 0.5
// (Abramowitz and Stegun 26.2.23 rational approximation, |error| < 4.5e-4); used only
// to place a first threshold guess, never to decide membership.
__device__ __forceinline__ float normal_upper_quantile(float p) {
    const float t = sqrtf(-2.f * logf(p));
    return t - (2.515517f + t * (0.802853f + t * 0.010328f)) /
                   (1.f + t * (1.432788f + t * (0.189269f + t * 0.001308f)));
}

}  // namespace
}  // namespace hils
