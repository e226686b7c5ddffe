// Chunk scoring and top-K: "Hierarchical Sparse Attention Done Right" (picx.dev
// summary), Eq. 7 and Methodology 2 (s^_{i,c} = q~_i . k'_c / sqrt(d) + b'_c), and the
// rcap.io post's pseudocode figure (keep the top K chunks per query).
//
// Exact selection. The kept set must equal the top K of the float64 score
//   x_c = (sum_x q~_x k'_x) * scale + b'_c   (each product and sum rounded to float64,
//                                             in x order),
// ties going to the lower chunk index. Every eligible chunk first gets a float32
// screen value s_c with a rigorous error radius e_c:
//   |fl32(sum q k) - sum q k| <= (d+1) 2^-24 sum|q k| (fused multiply-adds), plus one
//   rounding of s = fma(dot, scale, b'); e_c doubles both terms,
//   e_c = scale * sum|q k| * (d+2) 2^-23 + |s_c| 2^-22,
// which also covers the float64 value's own (~1e-15 relative) deviation.
// With lo = s - e and hi = s + e (directed rounding), s_K / s_{K+1} the K-th and
// (K+1)-th largest screen values and e_max the largest radius:
//   chunk certainly out  if hi_c < s_K - e_max   (K chunks are certainly above it),
//   chunk certainly in   if lo_c > s_{K+1} + e_max (at most K-1 others can reach it),
// and only the remaining "band" chunks get the float64 value, which decides the
// remaining places. Band chunks are rare (a few per thousand queries on the
// near-uniform prefill scores), so the float64 work stays small.
//
// Layout of the work: a warp scores 128 chunks at a time (one lane per chunk, 4 per
// lane) against the query held in shared memory as float32, keeps a running exact
// top-K list, and merges it with the next 128. Many queries (prefill): one warp per
// query. Few queries with long contexts (decode): the chunk range of a query is
// split over several 8-warp CTAs; each CTA reduces its warps' lists, writes its
// exact top-K to the workspace, and the last CTA to arrive merges them.
#include <float.h>
#include <limits.h>
#include <math.h>

#include "hils_internal.cuh"

namespace hils {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
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
    const T *qr = static_cast<const T *>(q.qrow);
    const T *kr = static_cast<const T *>(q.khead) + (int64_t)c * q.kst;
    double acc = 0.0;
#pragma unroll 4
    for (int x = 0; x < D; ++x) acc = __dadd_rn(acc, __dmul_rn(to_double(qr[x]), to_double(kr[x])));
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
template <typename T, int D, int R>
__device__ unsigned warp_topk(Slots<R> &p, int K, const QueryCtx &q, float &bound) {
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
template <typename T, int D>
__device__ void warp_scan(const QueryCtx &q, const float *qs, int c0, int c1, int K, EntryList &list) {
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
template <typename T, int D, int R>
__device__ void warp_merge(const QueryCtx &q, const EntryList *lists, int nlists, bool from_global, int K,
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
        for (int j = 0; j < n; ++j) rank += list.idx[j] < me;
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
    const int i = (int)(qi % a.Lq);
    const int h = (int)((qi / a.Lq) % a.H);
    const int b = (int)(qi / ((int64_t)a.Lq * a.H));
    t = a.qpos ? a.qpos[(int64_t)b * a.Lq + i] : i;
    QueryCtx q;
    q.qrow = static_cast<const T *>(a.Qcal.ptr) + b * a.Qcal.sb + h * a.Qcal.sh + i * a.Qcal.st;
    q.khead = static_cast<const T *>(a.Ksum.ptr) + b * a.Ksum.sb + h * a.Ksum.sh;
    q.kst = a.Ksum.st;
    q.bhead = a.Bsum + ((int64_t)b * a.H + h) * a.C;
    q.scale = a.scale;
    return q;
}

__device__ __forceinline__ int eligible(int t, int C) {
    const int e = t >= 0 ? t / kChunk : 0;
    return e < C ? e : C;
}

template <typename T, int D>
__device__ void load_query_f32(const QueryCtx &q, float *qs) {
    const T *qr = static_cast<const T *>(q.qrow);
    for (int x = threadIdx.x & 31; x < D; x += 32) qs[x] = (float)qr[x];
}

// Many queries: one warp per query, direct output.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) select_warp_kernel(SelectArgs a) {
    __shared__ __align__(16) float qs_all[kWarps][D];
    __shared__ EntryList lists[kWarps];
    const int w = threadIdx.x >> 5;
    const int64_t qi = (int64_t)blockIdx.x * kWarps + w;
    const int64_t nq = (int64_t)a.B * a.H * a.Lq;
    if (qi >= nq) return;
    int t;
    const QueryCtx q = make_ctx<T, D>(a, qi, t);
    const int ne = eligible(t, a.C);
    load_query_f32<T, D>(q, qs_all[w]);
    __syncwarp();
    warp_scan<T, D>(q, qs_all[w], 0, ne, a.topk, lists[w]);
    warp_write(lists[w], a.topk, qi, a.idx, a.score, a.nsel);
}

// ---- decode-shaped search (few queries, long contexts): screen, then pick
//
// S1 select_screen_kernel: grid (chunk blocks of 256, queries), 128 threads. A
// coalesced stream over the summary rows: kTPR threads share a row (16 bytes each),
// every thread keeps its slice of q~ in registers, 8 row loads in flight per thread,
// partial dot and |k|^2 combined with xor-shuffles. It writes the screen value s_c
// and its radius e_c of every eligible chunk to the workspace. The radius uses the
// Cauchy-Schwarz form of the fused-multiply-add bound, doubled:
//   e_c = scale |q~| |k'_c| (d+2) 2^-23 + |s_c| 2^-22.
// S2 select_pick_kernel: one 1024-thread CTA per query holds the query's screen
// values in registers (16 per thread), finds a threshold T with K+1 <= #{s >= T} <= 64
// (a normal-quantile guess, then bisection over the ordered float keys: at most 32
// rounds, usually none), keeps the chunks with hi >= T - e_max (every chunk that can
// still be among the top K: the K-th largest lo is at least T - e_max), and one warp
// runs the exact interval top-K on those. Heavy ties (more than 64 candidates) fall
// back to folding the candidates in batches of 32, which is always exact.
// S2 is launched with programmatic dependent launch, so its launch overlaps S1's tail.

constexpr int kSplitThreads = 128;
constexpr int kSpan = 256;         // chunks per screen CTA
constexpr int kPickThreads = 1024;
constexpr int kPickItems = 16;     // screen values per pick thread: C <= 16384
constexpr int kPoolCap = 64;

template <typename T, int D>
struct ScanCfg {
    static constexpr int kEPV = Vec<T>::kN;             // elements per 16-byte load
    static constexpr int kTPR = D / kEPV;               // threads per summary row: 8, 16 or 32
    static constexpr int kRPS = kSplitThreads / kTPR;   // rows per step
    static constexpr int kSteps = kSpan / kRPS;
    static constexpr int kUnroll = kSteps < 8 ? kSteps : 8;
    static_assert(kSteps % kUnroll == 0, "span");
};

__device__ __forceinline__ float2 *screen_buffer(const SelectArgs &a, int64_t qi) {
    return static_cast<float2 *>(a.ws) + qi * a.C;
}

template <typename T, int D>
__global__ void __launch_bounds__(kSplitThreads) select_screen_kernel(SelectArgs a) {
    using Cfg = ScanCfg<T, D>;
    constexpr int kN = Vec<T>::kN;
    pdl_trigger();
    __shared__ float b_scr[kSpan];
    const int64_t qi = blockIdx.y;
    int t;
    const QueryCtx q = make_ctx<T, D>(a, qi, t);
    const int ne = eligible(t, a.C);
    const int base = blockIdx.x * kSpan;
    if (base >= ne) return;
    const int c1 = min(base + kSpan, ne);
    const int tid = threadIdx.x, col = tid % Cfg::kTPR, r0 = tid / Cfg::kTPR;
    float qv[kN];
    widen(__ldg(reinterpret_cast<const uint4 *>(q.qrow) + col), qv, T());
    float qn2 = 0.f;
#pragma unroll
    for (int i = 0; i < kN; ++i) qn2 = fmaf(qv[i], qv[i], qn2);
#pragma unroll
    for (int o = Cfg::kTPR / 2; o > 0; o >>= 1) qn2 += __shfl_xor_sync(kFull, qn2, o);
    for (int i = tid; i < kSpan; i += kSplitThreads) {
        const int c = base + i;
        b_scr[i] = c < c1 ? q.bhead[c] : 0.f;
    }
    __syncthreads();
    float2 *out = screen_buffer(a, qi);
    const T *kh = static_cast<const T *>(q.khead);
    const float ecoef = q.scale * sqrtf(qn2) * ((float)(D + 2) * 0x1p-23f);
    for (int s0 = 0; s0 < Cfg::kSteps; s0 += Cfg::kUnroll) {
        uint4 v[Cfg::kUnroll];
#pragma unroll
        for (int u = 0; u < Cfg::kUnroll; ++u) {
            const int c = base + (s0 + u) * Cfg::kRPS + r0;
            v[u] = c < c1 ? __ldg(reinterpret_cast<const uint4 *>(kh + (int64_t)c * q.kst) + col)
                          : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < Cfg::kUnroll; ++u) {
            float kf[kN];
            widen(v[u], kf, T());
            float dot = 0.f, ksq = 0.f;
#pragma unroll
            for (int i = 0; i < kN; ++i) {
                dot = fmaf(qv[i], kf[i], dot);
                ksq = fmaf(kf[i], kf[i], ksq);
            }
#pragma unroll
            for (int o = Cfg::kTPR / 2; o > 0; o >>= 1) {
                dot += __shfl_xor_sync(kFull, dot, o);
                ksq += __shfl_xor_sync(kFull, ksq, o);
            }
            const int row = (s0 + u) * Cfg::kRPS + r0;
            const int c = base + row;
            if (col == 0 && c < c1) {
                const float sv = fmaf(dot, q.scale, b_scr[row]);
                out[c] = make_float2(sv, fmaf(ecoef, sqrtf(ksq), fabsf(sv) * 0x1p-22f));
            }
        }
    }
}

// Staging area for the candidate pool.
struct Pool64 {
    double x[kPoolCap];
    int idx[kPoolCap];
    float s[kPoolCap];
    float e[kPoolCap];
};

// Block-wide sum / max / min over the pick CTA (all threads call; result everywhere).
template <int kOp>  // 0 sum, 1 max, 2 min
__device__ __forceinline__ float block_reduce_f(float v, float *scratch) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float x = __shfl_xor_sync(kFull, v, o);
        v = kOp == 0 ? v + x : (kOp == 1 ? fmaxf(v, x) : fminf(v, x));
    }
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) scratch[w] = v;
    __syncthreads();
    v = scratch[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float x = __shfl_xor_sync(kFull, v, o);
        v = kOp == 0 ? v + x : (kOp == 1 ? fmaxf(v, x) : fminf(v, x));
    }
    return v;
}

__device__ __forceinline__ int block_sum_i(int v, int *scratch) {
    v = __reduce_add_sync(kFull, v);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) scratch[w] = v;
    __syncthreads();
    return __reduce_add_sync(kFull, scratch[lane]);
}

// Upper normal quantile z with P(Z > z) = p (0 < p < 0.5): the rational approximation
// of Abramowitz & Stegun 26.2.23 (|error| < 4.5e-4). Only a starting guess here.
__device__ __forceinline__ float normal_upper_quantile(float p) {
    const float t = sqrtf(-2.f * logf(p));
    return t - (2.515517f + t * (0.802853f + t * 0.010328f)) /
                   (1.f + t * (1.432788f + t * (0.189269f + t * 0.001308f)));
}

template <typename T, int D>
__global__ void __launch_bounds__(kPickThreads) select_pick_kernel(SelectArgs a) {
    __shared__ float fscr[32];
    __shared__ int iscr[32];
    __shared__ Pool64 pool;
    __shared__ EntryList out;
    pdl_wait();     // the screen grid has completed and its writes are visible
    pdl_trigger();  // let the next dependent-launched kernel be scheduled
    const int64_t qi = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    int t;
    const QueryCtx q = make_ctx<T, D>(a, qi, t);
    const int ne = eligible(t, a.C);
    const int K = a.topk;
    const float2 *scr = screen_buffer(a, qi);
    if (ne <= K) {  // every eligible chunk is kept, in index order
        for (int r = tid; r < K; r += kPickThreads) {
            a.idx[qi * K + r] = r < ne ? r : -1;
            a.score[qi * K + r] = r < ne ? __ldcg(&scr[r]).x : -INFINITY;
        }
        if (tid == 0) a.nsel[qi] = ne;
        return;
    }
    float sv[kPickItems], ev[kPickItems];
    float emax = 0.f, smax = -INFINITY, smin = INFINITY, sum = 0.f, sum2 = 0.f;
#pragma unroll
    for (int j = 0; j < kPickItems; ++j) {
        const int c = tid + j * kPickThreads;
        const float2 v = c < ne ? __ldcg(&scr[c]) : make_float2(-INFINITY, 0.f);
        sv[j] = v.x;
        ev[j] = v.y;
        if (c < ne) {
            emax = fmaxf(emax, v.y);
            smax = fmaxf(smax, v.x);
            smin = fminf(smin, v.x);
            sum += v.x;
            sum2 = fmaf(v.x, v.x, sum2);
        }
    }
    emax = block_reduce_f<1>(emax, fscr);
    smax = block_reduce_f<1>(smax, fscr);
    smin = block_reduce_f<2>(smin, fscr);
    sum = block_reduce_f<0>(sum, fscr);
    sum2 = block_reduce_f<0>(sum2, fscr);

    // threshold over ordered keys: invariant count(>= lo_key) >= K+1, count(>= hi_key) <= K
    unsigned lo_key = ordered_key(smin), hi_key = ordered_key(smax) + 1u;
    unsigned tk;
    {
        const float mu = sum / ne;
        const float sd = sqrtf(fmaxf(sum2 / ne - mu * mu, 0.f));
        const float p = fminf((float)(K + 8) / (float)ne, 0.49f);
        const float guess = mu + normal_upper_quantile(p) * sd;
        tk = min(max(ordered_key(guess), lo_key), hi_key - 1u);
    }
    for (int it = 0; it < 40; ++it) {
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < kPickItems; ++j) cnt += ordered_key(sv[j]) >= tk && sv[j] != -INFINITY;
        cnt = block_sum_i(cnt, iscr);
        if (cnt > kPoolCap) lo_key = tk;
        else if (cnt < K + 1) hi_key = tk;
        else break;
        if (hi_key - lo_key <= 1u) {
            tk = lo_key;
            break;
        }
        tk = lo_key + (hi_key - lo_key) / 2u;
    }
    // candidates: hi >= T - e_max
    const float cut = __fsub_rd(key_to_float(tk), emax);
    int mine = 0;
#pragma unroll
    for (int j = 0; j < kPickItems; ++j) mine += sv[j] != -INFINITY && __fadd_ru(sv[j], ev[j]) >= cut;
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
    }
    __syncthreads();
    if (lane == 31) iscr[w] = incl;
    __syncthreads();
    int wbase = 0;
    for (int k = 0; k < w; ++k) wbase += iscr[k];
    int total = 0;
    for (int k = 0; k < kPickThreads / 32; ++k) total += iscr[k];
    if (total <= kPoolCap) {
        int pos = wbase + incl - mine;
#pragma unroll
        for (int j = 0; j < kPickItems; ++j) {
            if (sv[j] != -INFINITY && __fadd_ru(sv[j], ev[j]) >= cut) {
                pool.idx[pos] = tid + j * kPickThreads;
                pool.s[pos] = sv[j];
                pool.e[pos] = ev[j];
                pool.x[pos] = __longlong_as_double(0x7ff8000000000000ll);
                ++pos;
            }
        }
        __syncthreads();
        if (w == 0) {
            Slots<2> p;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                const bool ok = j < total;
                p.idx[r] = ok ? pool.idx[j] : -1;
                p.s[r] = ok ? pool.s[j] : 0.f;
                p.e[r] = ok ? pool.e[j] : 0.f;
                p.x[r] = ok ? pool.x[j] : 0.0;
            }
            float bnd;
            const unsigned keep = warp_topk<T, D, 2>(p, K, q, bnd);
            __syncwarp();
            const int n = warp_append<2>(p, keep, out, 0);
            if (lane == 0) out.n = n;
            __syncwarp();
            warp_write(out, K, qi, a.idx, a.score, a.nsel);
        }
        return;
    }
    // heavy ties: fold the candidates in index order, 32 at a time (slot 0 = running list)
    if (w == 0) {
        int n = 0;
        for (int c0 = 0; c0 < ne; c0 += 32) {
            const int c = c0 + lane;
            const float2 v = c < ne ? __ldcg(&scr[c]) : make_float2(-INFINITY, 0.f);
            const bool cand = c < ne && __fadd_ru(v.x, v.y) >= cut;
            if (!__any_sync(kFull, cand)) continue;
            Slots<2> p;
            p.idx[0] = lane < n ? out.idx[lane] : -1;
            p.s[0] = lane < n ? out.s[lane] : 0.f;
            p.e[0] = lane < n ? out.e[lane] : 0.f;
            p.x[0] = lane < n ? out.x[lane] : 0.0;
            p.idx[1] = cand ? c : -1;
            p.s[1] = v.x;
            p.e[1] = v.y;
            p.x[1] = __longlong_as_double(0x7ff8000000000000ll);
            float bnd;
            const unsigned keep = warp_topk<T, D, 2>(p, K, q, bnd);
            __syncwarp();
            n = warp_append<2>(p, keep, out, 0);
            __syncwarp();
        }
        if (lane == 0) out.n = n;
        __syncwarp();
        warp_write(out, K, qi, a.idx, a.score, a.nsel);
    }
}

template <typename T, int D>
hils_status launch(const SelectArgs &a, cudaStream_t s) {
    const int64_t nq = (int64_t)a.B * a.H * a.Lq;
    if (nq == 0) return HILS_OK;
    if (a.ctas_per_query == 0) {
        const int64_t grid = (nq + kWarps - 1) / kWarps;
        select_warp_kernel<T, D><<<(unsigned)grid, kThreads, 0, s>>>(a);
    } else {
        select_screen_kernel<T, D><<<dim3(a.ctas_per_query, (unsigned)nq), kSplitThreads, 0, s>>>(a);
        const hils_status st = record_cuda_error(cudaGetLastError());
        if (st != HILS_OK) return st;
        return launch_dependent((const void *)select_pick_kernel<T, D>, dim3((unsigned)nq), dim3(kPickThreads),
                                0, s, a);
    }
    return record_cuda_error(cudaGetLastError());
}

}  // namespace

void select_split_plan(int B, int H, int Lq, int C, int K, bool has_qpos, int num_sms,
                       int *ctas_per_query, int *tiles_per_warp) {
    (void)has_qpos;
    (void)K;
    const int64_t nq = (int64_t)B * H * Lq;
    *tiles_per_warp = (C + kTile - 1) / kTile;
    // many queries, short tables, or tables beyond the pick kernel's register capacity:
    // one warp per query; otherwise screen + pick
    if (nq >= (int64_t)kWarps * num_sms || C <= kTile || C > kPickThreads * kPickItems || nq > 65535) {
        *ctas_per_query = 0;
        return;
    }
    *ctas_per_query = (C + kSpan - 1) / kSpan;
}

size_t select_ws_bytes(int queries, int C, int ctas_per_query) {
    if (ctas_per_query <= 0) return 0;
    return (size_t)queries * C * sizeof(float2);  // screen values and radii
}

hils_status launch_select(hils_dtype dt, int d, const SelectArgs &a, cudaStream_t s) {
    if (dt == HILS_BF16) return d == 64 ? launch<bf16, 64>(a, s) : launch<bf16, 128>(a, s);
    return d == 64 ? launch<float, 64>(a, s) : launch<float, 128>(a, s);
}

}  // namespace hils
