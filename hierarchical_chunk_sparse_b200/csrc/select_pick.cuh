// Exact top-K pick of one decode query, or of one (b, group, query) for grouped heads
// (summary page, Methodology 3), from the screen values of the decode select ("Hierarchical
// Sparse Attention Done Right" (picx.dev summary), Eq. 7 and Methodology 2; rcap.io post,
// pseudocode figure), for the decode select's pick kernel.
//
// Workspace of the decode select: a 256-byte status header, then the screen value and
// radius (s_c, e_c) of every eligible chunk per query, then the largest s and e of every
// 64-chunk group per query.
#pragma once
#include "select_common.cuh"

namespace hils {
namespace {

constexpr int kGroupRows = 64;  // rows per group maximum
constexpr int kMaxDecC = 16384; // table rows per query on this path
constexpr int kMaxGroups = kMaxDecC / kGroupRows;  // 256
constexpr int kPoolCap = 64;

// Staging area for the candidate pool.
struct Pool64 {
    double x[kPoolCap];
    int idx[kPoolCap];
    float s[kPoolCap];
    float e[kPoolCap];
};



// (K+1)-th largest of n <= kMaxGroups values (duplicates counted) from their
// order-preserving integer keys key[0..n), padded with zeros to a multiple of 4: value i
// has the unique rank #{j: k_j > k_i} + #{j < i: k_j = k_i}, and the one of rank K is
// the answer (n > K; all NT threads call; the result in *out). Two threads share a key,
// each counting over half of the keys (read four at a time by every thread at once, a
// broadcast), and add their counts with one shuffle.
template <int NT>
__device__ void block_kth_plus_one(const unsigned *key, int n, int K, float *out) {
    const uint4 *k4 = reinterpret_cast<const uint4 *>(key);
    const int n4 = (n + 3) >> 2, h4 = (n4 + 1) >> 1;
    const int half = threadIdx.x & 1;
    const int j4lo = half ? h4 : 0, j4hi = half ? n4 : h4;
    for (int i0 = 0; i0 < n; i0 += NT / 2) {  // uniform over the CTA: the shuffle needs every lane
        const int i = i0 + (threadIdx.x >> 1);
        const unsigned ki = i < n ? key[i] : 0u;
        int gt = 0, eq = 0;
#pragma unroll 4
        for (int j4 = j4lo; j4 < j4hi; ++j4) {
            const uint4 k = k4[j4];
            const int j = 4 * j4;
            gt += (k.x > ki) + (k.y > ki) + (k.z > ki) + (k.w > ki);
            eq += (k.x == ki && j < i) + (k.y == ki && j + 1 < i) + (k.z == ki && j + 2 < i) + (k.w == ki && j + 3 < i);
        }
        gt += __shfl_xor_sync(kFull, gt, 1);
        eq += __shfl_xor_sync(kFull, eq, 1);
        if (i < n && half == 0 && gt + eq == K) *out = key_to_float(ki);
    }
}

// The float64 score of chunk c for one query head, the same fixed-order chain as
// exact_score (each product of the float64 values, summed in x order, then times scale
// plus b'_c), with the query's elements from shared memory (float32 copies that hold
// the input values exactly).
template <typename T, int D>
__device__ __forceinline__ double exact_row(const QueryCtx &q, const float *qs, int c) {
    constexpr int kN = Vec<T>::kN, kHalf = D / kN / 2;
    const uint4 *kr = reinterpret_cast<const uint4 *>(static_cast<const T *>(q.khead) + (int64_t)c * q.kst);
    const float bias = __ldg(q.bhead + c);
    double acc = 0.0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint4 kv[kHalf];
#pragma unroll
        for (int u = 0; u < kHalf; ++u) kv[u] = __ldg(kr + h * kHalf + u);
#pragma unroll
        for (int u = 0; u < kHalf; ++u) {
            float kf[kN];
            widen(kv[u], kf, T());
#pragma unroll
            for (int i = 0; i < kN; ++i)
                acc = __dadd_rn(acc, __dmul_rn((double)qs[(h * kHalf + u) * kN + i], (double)kf[i]));
        }
    }
    return __dadd_rn(__dmul_rn(acc, (double)q.scale), (double)bias);
}

struct PickSmem {
    float qs[kMaxGroup * 128];  // the query rows (float32) of the unit's heads
    double xh[kMaxGroup * kPoolCap];  // float64 score of each (head, pool entry)
    uint8_t kept[kPoolCap];
    float2 gm[kMaxGroups];
    __align__(16) unsigned gkey[kMaxGroups];  // order-preserving keys of gm[].x
    uint16_t cand_g[kMaxGroups];
    Pool64 pool;
    EntryList out;
    float wmax[8];  // one per warp of the picking CTA
    float cut, tk;
    int ncg, pool_n;
};

struct ScreenWs {
    float2 *scr;   // [queries][C]
    float2 *gmax;  // [queries][ceil(C/64)]
};

__host__ __device__ __forceinline__ int groups_of(int C) { return (C + kGroupRows - 1) / kGroupRows; }

__host__ __device__ __forceinline__ size_t dec_ws_bytes(int64_t queries, int C) {
    const size_t scr = (size_t)queries * (C + groups_of(C)) * sizeof(float2);
    return kSelectStatusBytes + scr;
}

// The screen row one pick unit reads (one query's, or the group centres and radii the
// screen folded for a (b, group, query)), and its 64-chunk maxima.
struct ScrRows {
    const float2 *scr, *gmx;
};

__device__ __forceinline__ ScreenWs screen_ws(const SelectArgs &a) {
    const int64_t nq = (int64_t)a.B * a.H * a.Lq;
    ScreenWs w;
    w.scr = reinterpret_cast<float2 *>(static_cast<uint8_t *>(a.ws) + kSelectStatusBytes);
    w.gmax = w.scr + nq * a.C;
    return w;
}

// Exact top-K of one unit from the screen values in the workspace (all NT threads of
// a CTA, NT <= 256; every step below is one parallel round trip to L2). A unit is one
// query (kGroup = false) or, for grouped heads, one (b, group, query) whose chunks are
// ranked by the maximum over the group's heads of their scores.
template <typename T, int D, int NT, bool kGroup>
__device__ void pick_unit(const SelectArgs &a, const ScreenWs &ws, int64_t u, PickSmem &ps) {
    using Ctx = std::conditional_t<kGroup, GroupCtx, QueryCtx>;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    int t, b = 0, grp = 0, i = 0;
    Ctx q;
    ScrRows rows;
    if constexpr (kGroup) {
        q = make_group_ctx<T, D>(a, u, t, b, grp, i);
        for (int hh = 0; hh < a.G; ++hh)
            for (int x = tid; x < D; x += NT)
                ps.qs[hh * D + x] = (float)static_cast<const T *>(q.head.qrow)[hh * q.qsh + x];
    } else {
        q = make_ctx<T, D>(a, u, t);
        for (int x = tid; x < D; x += NT) ps.qs[x] = (float)static_cast<const T *>(q.qrow)[x];
    }
    rows.scr = ws.scr + u * a.C;
    rows.gmx = ws.gmax + u * groups_of(a.C);
    auto write = [&](const EntryList &list) {
        if constexpr (kGroup) group_write<T, D>(q, ps.qs, list, a, u, b, grp, i);
        else warp_write(list, a.topk, u, a.idx, a.score, a.nsel);
    };
    const int ne = eligible(t, a.C, a.excl_w);
    const int K = a.topk;
    if (ne <= K) {  // every eligible chunk is kept, in index order
        if constexpr (kGroup) {
            __syncthreads();  // ps.qs complete
            if (w == 0) {
                if (lane < ne) ps.out.idx[lane] = lane;
                if (lane == 0) ps.out.n = ne;
                __syncwarp();
                write(ps.out);
            }
        } else {
            for (int r = tid; r < K; r += NT) {
                a.idx[u * K + r] = r < ne ? r : -1;
                a.score[u * K + r] = r < ne ? __ldcg(&rows.scr[r]).x : -INFINITY;
            }
            if (tid == 0) a.nsel[u] = ne;
        }
        return;
    }
    const int G = groups_of(ne);
    if (G < K + 1) {  // short table: the exact running-list scan over every chunk
        __syncthreads();  // ps.qs complete
        if (w == 0) {
            warp_scan<T, D>(q, ps.qs, 0, ne, K, ps.out);
            write(ps.out);
        }
        return;
    }
    // T = (K+1)-th largest maximum of the 64-chunk groups (attained by K+1 distinct
    // chunks); e_max = largest radius; every chunk with hi < T - e_max is certainly out
    float em = 0.f;
    for (int g = tid; g < ((G + 3) & ~3); g += NT) {
        const float2 v = g < G ? __ldcg(&rows.gmx[g]) : make_float2(-INFINITY, 0.f);
        ps.gm[g] = v;
        ps.gkey[g] = g < G ? ordered_key(v.x) : 0u;  // 0: below every value's key
        em = fmaxf(em, v.y);
    }
    em = warp_max(em);
    if (tid == 0) {
        ps.ncg = 0;
        ps.pool_n = 0;
    }
    if (lane == 0) ps.wmax[w] = em;
    __syncthreads();  // ps.qs, ps.gm and ps.gkey complete
    block_kth_plus_one<NT>(ps.gkey, G, K, &ps.tk);
    __syncthreads();
    if (tid == 0) {
        float e2 = 0.f;
        for (int k = 0; k < NT / 32; ++k) e2 = fmaxf(e2, ps.wmax[k]);
        ps.cut = __fsub_rd(ps.tk, e2);
    }
    __syncthreads();
    const float cut = ps.cut;
    // candidate groups: their max s + max e can reach the cut
    for (int g = tid; g < G; g += NT)
        if (__fadd_ru(ps.gm[g].x, ps.gm[g].y) >= cut) ps.cand_g[atomicAdd(&ps.ncg, 1)] = (uint16_t)g;
    __syncthreads();
    const int ncg = ps.ncg;
    // their chunks with hi >= cut join the pool: slot e of the candidates' chunks is
    // chunk e % 64 of candidate group e / 64; a thread loads its (up to) eight slots at
    // once
    constexpr int kPer = 8;
    for (int e0 = 0; e0 < ncg * kGroupRows; e0 += NT * kPer) {
        float2 v[kPer];
        int cc[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = e0 + j * NT + tid;
            cc[j] = e < ncg * kGroupRows ? ps.cand_g[e / kGroupRows] * kGroupRows + e % kGroupRows : ne;
            v[j] = cc[j] < ne ? __ldcg(&rows.scr[cc[j]]) : make_float2(-INFINITY, 0.f);
        }
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            if (v[j].x != -INFINITY && __fadd_ru(v[j].x, v[j].y) >= cut) {
                const int pos = atomicAdd(&ps.pool_n, 1);
                if (pos < kPoolCap) {
                    ps.pool.idx[pos] = cc[j];
                    ps.pool.s[pos] = v[j].x;
                    ps.pool.e[pos] = v[j].y;
                    ps.pool.x[pos] = __longlong_as_double(0x7ff8000000000000ll);
                }
            }
        }
    }
    __syncthreads();  // every candidate is in the pool before any thread reads it
    const int total = ps.pool_n;
    if constexpr (!kGroup) {
      if (total <= kPoolCap) {
        // the candidates' screen values carry the fused-multiply-add radius already, so
        // few need the float64 score
        if (w == 0) {
            Slots<2> sl;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int j = lane + 32 * r;
                const bool ok = j < total;
                sl.idx[r] = ok ? ps.pool.idx[j] : -1;
                sl.s[r] = ok ? ps.pool.s[j] : 0.f;
                sl.e[r] = ok ? ps.pool.e[j] : 0.f;
                sl.x[r] = ok ? ps.pool.x[j] : 0.0;
            }
            float bnd;
            const unsigned keep = warp_topk<T, D, 2>(sl, K, q, bnd);
            __syncwarp();
            const int n = warp_append<2>(sl, keep, ps.out, 0);
            if (lane == 0) ps.out.n = n;
            __syncwarp();
            write(ps.out);
        }
        return;
      }
    } else if (total <= kPoolCap) {
        // Grouped heads: every chunk outside the pool is certainly out, and the pool
        // holds more than K chunks (the K+1 that attain the largest group maxima). The
        // float64 score of every (head, pool entry), one thread each, decides the kept
        // set exactly: the K largest by (score, then lower chunk index); a group's score
        // is the largest of its heads'.
        const int nh = a.G;
        for (int p = tid; p < total * nh; p += NT) {
            const int j = p % total, hh = p / total;
            ps.xh[hh * kPoolCap + j] = exact_row<T, D>(head_ctx(q, hh, (int)sizeof(T)), ps.qs + hh * D, ps.pool.idx[j]);
        }
        __syncthreads();
        for (int j = tid; j < total; j += NT) {
            double x = ps.xh[j];
            for (int hh = 1; hh < nh; ++hh) x = fmax(x, ps.xh[hh * kPoolCap + j]);
            ps.pool.x[j] = x;
        }
        __syncthreads();
        for (int j = tid; j < total; j += NT) {
            const double xj = ps.pool.x[j];
            const int cj = ps.pool.idx[j];
            int rank = 0;
            for (int k = 0; k < total; ++k) {
                const double xk = ps.pool.x[k];
                rank += (xk > xj || (xk == xj && ps.pool.idx[k] < cj)) ? 1 : 0;
            }
            ps.kept[j] = rank < K ? 1 : 0;
        }
        __syncthreads();
        // outputs in ascending chunk index: each kept entry's position is the number of
        // kept entries with a lower index; scores are the heads' own (rounded) values
        for (int j = tid; j < total; j += NT) {
            if (!ps.kept[j]) continue;
            const int cj = ps.pool.idx[j];
            int pos = 0;
            for (int k = 0; k < total; ++k) pos += (ps.kept[k] && ps.pool.idx[k] < cj) ? 1 : 0;
            a.idx[u * K + pos] = cj;
            for (int hh = 0; hh < a.G; ++hh)
                a.score[(((int64_t)b * a.H + grp * a.G + hh) * a.Lq + i) * K + pos] = (float)ps.xh[hh * kPoolCap + j];
        }
        if (tid == 0) a.nsel[u] = K;
        return;
    }
    if (w != 0) return;
    // heavy ties: fold the candidates in index order, 32 at a time (slot 0 = running list)
    int n = 0;
    for (int c0 = 0; c0 < ne; c0 += 32) {
        const int c = c0 + lane;
        const float2 v = c < ne ? __ldcg(&rows.scr[c]) : make_float2(-INFINITY, 0.f);
        const bool cand = c < ne && __fadd_ru(v.x, v.y) >= cut;
        if (!__any_sync(kFull, cand)) continue;
        Slots<2> sl;
        sl.idx[0] = lane < n ? ps.out.idx[lane] : -1;
        sl.s[0] = lane < n ? ps.out.s[lane] : 0.f;
        sl.e[0] = lane < n ? ps.out.e[lane] : 0.f;
        sl.x[0] = lane < n ? ps.out.x[lane] : 0.0;
        sl.idx[1] = cand ? c : -1;
        sl.s[1] = v.x;
        sl.e[1] = v.y;
        sl.x[1] = __longlong_as_double(0x7ff8000000000000ll);
        float bnd;
        const unsigned keep = warp_topk<T, D, 2>(sl, K, q, bnd);
        __syncwarp();
        n = warp_append<2>(sl, keep, ps.out, 0);
        __syncwarp();
    }
    if (lane == 0) ps.out.n = n;
    __syncwarp();
    write(ps.out);
}

}  // namespace
}  // namespace hils
