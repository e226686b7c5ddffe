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
template <typename T, int D, int R>
__device__ unsigned warp_topk(Slots<R> &p, int K, const QueryCtx &q) {
    const int lane = threadIdx.x & 31;
    unsigned valid = 0;
#pragma unroll
    for (int r = 0; r < R; ++r)
        if (p.idx[r] >= 0) valid |= 1u << r;
    const int n = __reduce_add_sync(kFull, __popc(valid));
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
        const unsigned keep = warp_topk<T, D, 5>(p, K, q);
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
    const unsigned keep = warp_topk<T, D, R>(p, K, q);
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

// ---- split search (few queries, long contexts)
//
// A CTA screens its chunk range in passes of 1024 chunks. The screen is a coalesced
// stream over the summary rows: kTPR threads share a row (16 B each), every thread
// keeps its slice of q~ in registers and has kUnroll row loads in flight; the row's
// partial dot / |dot| are combined with xor-shuffles. Screen values and radii land in
// shared memory, and then each warp folds its 128 of them into its running exact
// top-K list exactly as the per-query path does.

template <typename T, int D>
struct ScanCfg {
    static constexpr int kEPV = Vec<T>::kN;       // elements per 16-byte load
    static constexpr int kTPR = D / kEPV;         // threads per summary row: 8, 16 or 32
    static constexpr int kRPS = kThreads / kTPR;  // rows per step
    static constexpr int kPass = kWarps * kTile;  // 1024 chunks per pass
    static constexpr int kSteps = kPass / kRPS;
    static constexpr int kUnroll = 16;
    static_assert(kSteps % kUnroll == 0, "pass size");
};

template <typename T, int D>
__device__ void cta_screen_pass(const QueryCtx &q, const float (&qv)[Vec<T>::kN], int base, int c1,
                                float *s_scr, float *e_scr, float *b_scr) {
    using Cfg = ScanCfg<T, D>;
    constexpr int kN = Vec<T>::kN;
    const int tid = threadIdx.x, col = tid % Cfg::kTPR, r0 = tid / Cfg::kTPR;
    for (int i = tid; i < Cfg::kPass; i += kThreads) {
        const int c = base + i;
        b_scr[i] = c < c1 ? q.bhead[c] : 0.f;
    }
    __syncthreads();
    const T *kh = static_cast<const T *>(q.khead);
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
            float dot = 0.f, ad = 0.f;
#pragma unroll
            for (int i = 0; i < kN; ++i) {
                dot = fmaf(qv[i], kf[i], dot);
                ad = fmaf(fabsf(qv[i]), fabsf(kf[i]), ad);
            }
#pragma unroll
            for (int o = Cfg::kTPR / 2; o > 0; o >>= 1) {
                dot += __shfl_xor_sync(kFull, dot, o);
                ad += __shfl_xor_sync(kFull, ad, o);
            }
            const int row = (s0 + u) * Cfg::kRPS + r0;
            if (col == 0) {
                const float sv = fmaf(dot, q.scale, b_scr[row]);
                s_scr[row] = sv;
                e_scr[row] = fmaf(q.scale * ad, (float)(D + 2) * 0x1p-23f, fabsf(sv) * 0x1p-22f);
            }
        }
    }
    __syncthreads();
}

// Folds the warp's 128 screened chunks of the pass into its running list.
template <typename T, int D>
__device__ int warp_fold(const QueryCtx &q, const float *s_scr, const float *e_scr, int base, int c1, int K,
                         EntryList &list, int n) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    Slots<5> p;
    p.idx[0] = lane < n ? list.idx[lane] : -1;
    p.s[0] = lane < n ? list.s[lane] : 0.f;
    p.e[0] = lane < n ? list.e[lane] : 0.f;
    p.x[0] = lane < n ? list.x[lane] : 0.0;
#pragma unroll
    for (int r = 1; r < 5; ++r) {
        const int row = w * kTile + lane + 32 * (r - 1);
        const int c = base + row;
        const bool ok = c < c1;
        p.idx[r] = ok ? c : -1;
        p.s[r] = ok ? s_scr[row] : 0.f;
        p.e[r] = ok ? e_scr[row] : 0.f;
        p.x[r] = __longlong_as_double(0x7ff8000000000000ll);
    }
    const unsigned keep = warp_topk<T, D, 5>(p, K, q);
    __syncwarp();
    n = warp_append<5>(p, keep, list, 0);
    __syncwarp();
    return n;
}

// Few queries, many chunks: grid (ctas_per_query, queries).
template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2) select_split_kernel(SelectArgs a) {
    using Cfg = ScanCfg<T, D>;
    __shared__ float s_scr[Cfg::kPass], e_scr[Cfg::kPass], b_scr[Cfg::kPass];
    __shared__ EntryList lists[kWarps];
    __shared__ EntryList merged;
    __shared__ int is_last;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t qi = blockIdx.y;
    int t;
    const QueryCtx q = make_ctx<T, D>(a, qi, t);
    const int ne = eligible(t, a.C);
    float qv[Vec<T>::kN];
    {
        float tmp[Vec<T>::kN];
        const int col = threadIdx.x % Cfg::kTPR;
        widen(__ldg(reinterpret_cast<const uint4 *>(q.qrow) + col), tmp, T());
#pragma unroll
        for (int i = 0; i < Vec<T>::kN; ++i) qv[i] = tmp[i];
    }
    int n = 0;
    for (int pass = 0; pass < a.tiles_per_warp; ++pass) {
        const int base = (blockIdx.x * a.tiles_per_warp + pass) * Cfg::kPass;
        if (base >= ne) break;
        const int c1 = min(base + Cfg::kPass, ne);
        cta_screen_pass<T, D>(q, qv, base, c1, s_scr, e_scr, b_scr);
        n = warp_fold<T, D>(q, s_scr, e_scr, base, c1, a.topk, lists[w], n);
        __syncthreads();
    }
    if (lane == 0) lists[w].n = n;
    __syncthreads();
    if (w == 0) warp_merge<T, D, 8>(q, lists, kWarps, false, a.topk, merged);
    __syncthreads();

    if (gridDim.x == 1) {
        if (w == 0) warp_write(merged, a.topk, qi, a.idx, a.score, a.nsel);
        return;
    }
    // publish this CTA's list; the last CTA of the query merges all of them
    int *counters = static_cast<int *>(a.ws);
    EntryList *ws_lists = reinterpret_cast<EntryList *>(
        static_cast<uint8_t *>(a.ws) + (((size_t)gridDim.y * sizeof(int) + 255) & ~(size_t)255));
    EntryList &mine = ws_lists[qi * gridDim.x + blockIdx.x];
    if (w == 0) {
        if (lane < merged.n) {
            mine.idx[lane] = merged.idx[lane];
            mine.s[lane] = merged.s[lane];
            mine.e[lane] = merged.e[lane];
            mine.x[lane] = merged.x[lane];
        }
        if (lane == 0) mine.n = merged.n;
        __threadfence();
        __syncwarp();
        if (lane == 0) is_last = atomicAdd(&counters[qi], 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (w == 0) {
        warp_merge<T, D, 16>(q, &ws_lists[qi * gridDim.x], gridDim.x, true, a.topk, merged);
        warp_write(merged, a.topk, qi, a.idx, a.score, a.nsel);
        if (threadIdx.x == 0) counters[qi] = 0;
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
        select_split_kernel<T, D><<<dim3(a.ctas_per_query, (unsigned)nq), kThreads, 0, s>>>(a);
    }
    return record_cuda_error(cudaGetLastError());
}

}  // namespace

void select_split_plan(int B, int H, int Lq, int C, int K, bool has_qpos, int num_sms,
                       int *ctas_per_query, int *tiles_per_warp) {
    (void)has_qpos;
    const int64_t nq = (int64_t)B * H * Lq;
    *tiles_per_warp = 1;
    if (nq >= (int64_t)kWarps * num_sms || C <= kTile) {
        *ctas_per_query = 0;  // one warp per query
        *tiles_per_warp = (C + kTile - 1) / kTile;
        return;
    }
    const int k = K > 0 ? K : 1;
    int tpw = 1;  // 1024-chunk passes per CTA
    for (;;) {
        const int span = kWarps * kTile * tpw;
        const int ctas = (C + span - 1) / span;
        if (ctas * k <= 16 * 32) {
            *ctas_per_query = ctas;
            *tiles_per_warp = tpw;
            return;
        }
        ++tpw;
    }
}

size_t select_ws_bytes(int queries, int ctas_per_query, int K) {
    (void)K;
    if (ctas_per_query <= 1) return 0;
    const size_t counters = ((size_t)queries * sizeof(int) + 255) & ~(size_t)255;
    return counters + (size_t)queries * ctas_per_query * sizeof(EntryList);
}

hils_status launch_select(hils_dtype dt, int d, const SelectArgs &a, cudaStream_t s) {
    if (dt == HILS_BF16) return d == 64 ? launch<bf16, 64>(a, s) : launch<bf16, 128>(a, s);
    return d == 64 ? launch<float, 64>(a, s) : launch<float, 128>(a, s);
}

}  // namespace hils
