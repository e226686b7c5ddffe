// One decode step per query in one thread-block cluster: "Hierarchical Sparse Attention
// Done Right" (picx.dev summary), Eq. 7 (chunk scores), Methodology 2 and Eq. 10 (the
// hierarchical softmax over the kept chunks and the window), and the rcap.io post's
// pseudocode figure.
//
// A cluster of 8 CTAs (128 threads each) takes one query (b, h) at t = cache_len[b] - 1.
// CTA r of the cluster:
//   1. streams, through a 5-stage cp.async ring, first its window tiles (tile j with
//      j % 8 == r; K and V take one stage each) and then its eighth of the eligible
//      chunk summaries (64-row items). Window tiles are attended as they arrive;
//      summary rows are screened on the tensor cores (bf16) or CUDA cores (float32)
//      into screen values s_c with rigorous radii e_c, kept in shared memory, with the
//      largest s and e of every 64-chunk group;
//   2. after a cluster barrier reads every CTA's group maxima through distributed
//      shared memory and computes T = the (K+1)-th largest group maximum (attained by
//      K+1 distinct chunks) and e_max: every chunk with hi < T - e_max is certainly
//      out; it compacts its own remaining candidates;
//      each candidate (typically K + a few per query, spread over the CTAs) is screened
//      again on CUDA cores with the tight radius while its K and V rows are prefetched
//      into L2, and is handed to the leader (remote shared-memory stores);
//   3. (leader, r = 0) after a second barrier runs the exact interval top-K over the
//      candidates (float64 score only for the band), writes idx / score / nsel and hands
//      the kept list, ascending, to every CTA;
//   4. after a third barrier attends its share of the kept chunks (slots r, r+8, ...)
//      and folds every unit it attended into one running (max, sum, weighted vector);
//   5. after a fourth barrier the leader combines the 8 partials into o and lse.
// The kept chunks, their scores and o are those of hils_select followed by
// hils_attend_decode; no screen value or partial leaves the cluster. Short tables
// (fewer than K+1 groups) and heavy ties (more than 64 candidates) take the exact
// running-list scan of the other select paths in the leader.
#include <cooperative_groups.h>

#include "screen_stage.cuh"

namespace hils {
namespace {

namespace cg = cooperative_groups;

constexpr int kCl = 8;            // CTAs per cluster (one query)
constexpr int kClThreads = 128;   // threads per CTA
constexpr int kClRows = 64;       // summary rows per stage
constexpr int kClStages = 5;
constexpr int kClMaxLocal = 1024; // eligible chunks per CTA (C <= 8192): two CTAs fit one SM
constexpr int kClMaxLocalGroups = kClMaxLocal / kGroupRows;
constexpr int kPushCap = 24;      // candidates a CTA hands to the leader directly

template <typename T, int D>
struct ClCfg : StageCfg<T, D, kClThreads, kClRows> {
    using Base = StageCfg<T, D, kClThreads, kClRows>;
    static constexpr int kTileBytes = kChunk * Base::kRowBytes;  // one K or V tile of 64 rows
    static_assert(kTileBytes <= Base::kStageBytes, "a K or V tile fits one stage");
    static constexpr int kStageStride = (Base::kStageBytes + 127) & ~127;
};

// Shared memory besides the stage ring.
template <int D>
struct ClSmem {
    union {
        float2 scr[kClMaxLocal];       // this CTA's screen values (s, e), local index
        float part_acc[kCl][D];        // leader, after the pick: every CTA's weighted vector
    };
    float2 gmax[kClMaxLocalGroups];    // this CTA's group maxima
    float2 gall[kMaxGroups];           // every group maximum of the query (gathered)
    float2 gscr[16];                   // per-warp maxima of the current stage
    float qf[D];                       // the query row q (window and chunk units), float
    float qs[D];                       // the scoring query q~ (leader's rescreen), float
    float logit[kChunk], prob[kChunk];
    float red[2 * kClThreads];         // unit output columns, one row per row group
    float acc[D];                      // running weighted sum of unit outputs
    float run_m, run_z;                // running max and sum of the unit weights
    float cut, tk, lse_tile;
    int ncand;
    Pool64 cand;                       // this CTA's candidates (global chunk index, s, e)
    int prank[kPoolCap];               // leader: rank of each candidate
    Pool64 pool;                       // leader: all candidates
    int push_n[kCl];                   // leader: candidates of each CTA (written by that CTA)
    int push_idx[kCl][kPushCap];       // leader: their chunk indices and tight (s, e)
    float push_s[kCl][kPushCap], push_e[kCl][kPushCap];
    float part_m[kCl], part_z[kCl];    // leader: every CTA's running max and sum
    EntryList out;                     // leader: kept list (unsorted)
    int sel_n, sel_mode;               // leader: kept count; 0 normal, 1 short table or ties
    int sel_idx[kMaxK];                // leader: kept list, ascending chunk index
    float sel_s[kMaxK];
    float wmax[4];
};

// 16-byte cp.async copies of `rows` consecutive rows (row stride st elements) into a
// plain row-major tile.
template <typename T, int D>
__device__ __forceinline__ void tile_issue(uint8_t *dst, const T *src, int64_t st, int rows) {
    constexpr int kUnits = D * (int)sizeof(T) / 16;
    for (int i = threadIdx.x; i < rows * kUnits; i += kClThreads) {
        const int r = i / kUnits, un = i - r * kUnits;
        cp_async16(dst + i * 16, reinterpret_cast<const uint8_t *>(src + r * st) + un * 16);
    }
}

// One unit (64 or fewer keys of K and V in plain tiles): its softmax-weighted value
// sum_j p_j v_j into s.red[0..D) and the log-mass log sum_j exp(scale q.k_j) into
// s.lse_tile. Two threads per key row for the logits (16-byte units in an order rotated
// by the row, so that a warp's reads spread over the banks), one warp for the softmax,
// two row halves per output column.
template <typename T, int D>
__device__ void cl_unit(ClSmem<D> &s, const uint8_t *kt, const uint8_t *vt, int rows, float scale) {
    constexpr int kRowBytes = D * (int)sizeof(T);
    constexpr int kHalf = kRowBytes / 32;  // 16-byte units per half row
    const int tid = threadIdx.x;
    {
        const int row = tid >> 1, half = tid & 1;
        float acc = 0.f;
        if (row < rows) {
            const uint4 *kr = reinterpret_cast<const uint4 *>(kt + row * kRowBytes);
#pragma unroll
            for (int k = 0; k < kHalf; ++k) {
                const int un = half * kHalf + ((k + row) % kHalf);
                float kf[Vec<T>::kN];
                widen(kr[un], kf, T());
#pragma unroll
                for (int i = 0; i < Vec<T>::kN; ++i) acc = fmaf(s.qf[un * Vec<T>::kN + i], kf[i], acc);
            }
        }
        acc += __shfl_xor_sync(kFull, acc, 1);
        if (half == 0 && row < kChunk) s.logit[row] = row < rows ? acc * scale : -INFINITY;
    }
    __syncthreads();
    if (tid < 32) {
        const float l0 = s.logit[tid], l1 = s.logit[tid + 32];
        const float m = warp_max(fmaxf(l0, l1));
        const float e0 = expf(l0 - m), e1 = expf(l1 - m);
        const float z = warp_sum(e0 + e1);
        const float inv = 1.f / z;
        s.prob[tid] = e0 * inv;
        s.prob[tid + 32] = e1 * inv;
        if (tid == 0) s.lse_tile = m + logf(z);
    }
    __syncthreads();
    {
        // thread: column pair cp (D/2 pairs), row half rh (rows rh, rh+2, ...)
        constexpr int kPairs = D / 2;
        const int cp = tid % kPairs, rh = tid / kPairs;
        float a0 = 0.f, a1 = 0.f;
        for (int j = rh; j < rows; j += kClThreads / kPairs) {
            const float2 vv = load2(reinterpret_cast<const T *>(vt + j * kRowBytes) + 2 * cp);
            const float pj = s.prob[j];
            a0 = fmaf(pj, vv.x, a0);
            a1 = fmaf(pj, vv.y, a1);
        }
        s.red[rh * D + 2 * cp] = a0;
        s.red[rh * D + 2 * cp + 1] = a1;
    }
    __syncthreads();
}

// Folds a unit (log-mass m, output in s.red as row halves) into the CTA's running sum.
template <int D>
__device__ void cl_fold(ClSmem<D> &s, float m) {
    constexpr int kHalves = kClThreads / (D / 2);
    if (m == -INFINITY) return;
    const float M = s.run_m, Mn = fmaxf(M, m);
    const float fo = expf(M - Mn), fn = expf(m - Mn);  // fo = 0 when M is -inf
    for (int x = threadIdx.x; x < D; x += kClThreads) {
        float o = 0.f;
#pragma unroll
        for (int hh = 0; hh < kHalves; ++hh) o += s.red[hh * D + x];
        s.acc[x] = s.acc[x] * fo + fn * o;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        s.run_z = s.run_z * fo + fn;
        s.run_m = Mn;
    }
    __syncthreads();
}

template <typename T, int D>
__global__ void __cluster_dims__(kCl, 1, 1) __launch_bounds__(kClThreads) decode_cluster_kernel(SelectArgs sa,
                                                                                               AttendArgs aa) {
    using Cfg = ClCfg<T, D>;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ ClSmem<D> s;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t qi = blockIdx.y;  // (b, h), one query
    const int b = (int)(qi / sa.H), h = (int)(qi % sa.H);
    const int K = sa.topk;
    const int t = aa.cache_len[b] - 1;
    const int ne = eligible(t, sa.C);
    // this CTA's groups of eligible chunks (an item is one 64-chunk group)
    const int G = groups_of(ne);
    const int gper = (G + kCl - 1) / kCl;
    const int g0 = min(G, rank * gper), g1 = min(G, g0 + gper);
    const int c_begin = g0 * kGroupRows, nloc = max(0, min(ne, g1 * kGroupRows) - c_begin);
    const int nitems = g1 - g0;
    // this CTA's window tiles: j = rank, rank + 8, ...
    int w0 = 0, nwt = 0;
    if (aa.W > 0 && t >= 0) {
        w0 = max(0, t - aa.W + 1);
        nwt = (t - w0) / kChunk + 1;
    }
    const int my_wt = nwt > rank ? (nwt - rank + kCl - 1) / kCl : 0;
    const int nslots = 2 * my_wt + nitems;

    const T *kh = static_cast<const T *>(sa.Ksum.ptr) + b * sa.Ksum.sb + h * sa.Ksum.sh;
    const float *bh = sa.Bsum + ((int64_t)b * sa.H + h) * sa.C;
    const T *qcal = static_cast<const T *>(sa.Qcal.ptr) + b * sa.Qcal.sb + h * sa.Qcal.sh;
    const T *qrow = static_cast<const T *>(aa.Q.ptr) + b * aa.Q.sb + h * aa.Q.sh;
    const T *kc = static_cast<const T *>(aa.K.ptr) + b * aa.K.sb + h * aa.K.sh;
    const T *vc = static_cast<const T *>(aa.V.ptr) + b * aa.V.sb + h * aa.V.sh;
    auto stage = [&](int k) { return ring + (k % kClStages) * Cfg::kStageStride; };
    auto tile_rows = [&](int start) { return min(kChunk, t - start + 1); };

    for (int x = tid; x < D; x += kClThreads) {
        s.qf[x] = (float)qrow[x];
        s.qs[x] = (float)qcal[x];
        s.acc[x] = 0.f;
    }
    if (tid == 0) {
        s.run_m = -INFINITY;
        s.run_z = 0.f;
        s.ncand = 0;
        s.sel_n = 0;
        s.sel_mode = 0;
    }
    // slot k: window tile k/2 (K for even k, V for odd k), then summary item k - 2*my_wt
    auto issue = [&](int k) {
        if (k < nslots) {
            uint8_t *buf = stage(k);
            if (k < 2 * my_wt) {
                const int start = w0 + (rank + (k >> 1) * kCl) * kChunk;
                tile_issue<T, D>(buf, ((k & 1) ? vc : kc) + (int64_t)start * ((k & 1) ? aa.V.st : aa.K.st),
                                 (k & 1) ? aa.V.st : aa.K.st, tile_rows(start));
            } else {
                const int c0 = c_begin + (k - 2 * my_wt) * kClRows;
                stage_issue<T, Cfg>(buf, kh, sa.Ksum.st, c0, min(kClRows, c_begin + nloc - c0), bh + c0, qcal,
                                    nullptr, t);
            }
        }
        cp_async_commit();
    };
    for (int k = 0; k < kClStages - 1; ++k) issue(k);
    __syncthreads();  // the query rows and running state are initialised
    for (int k = 0; k < nslots; ++k) {
        cp_async_wait<kClStages - 2>();
        __syncthreads();
        if (k < 2 * my_wt) {
            if (k & 1) {  // K (slot k-1) and V (slot k) of a window tile are in
                const int start = w0 + (rank + (k >> 1) * kCl) * kChunk;
                cl_unit<T, D>(s, stage(k - 1), stage(k), tile_rows(start), aa.scale);
                cl_fold<D>(s, s.lse_tile);
            }
        } else {
            const int it = k - 2 * my_wt;
            if (Cfg::kMma) screen_stage_mma<D>(stage(k), Cfg::kQOff, Cfg::kBiasOff, sa.scale, it * kClRows, nloc, s.scr, s.gscr);
            else screen_stage_f32<T, D, Cfg>(stage(k), sa.scale, it * kClRows, nloc, s.scr, s.gscr);
            __syncthreads();
            if (tid == 0) {  // one item is one 64-chunk group
                float2 m = s.gscr[0];
                for (int j = 1; j < Cfg::kSlots; ++j) {
                    m.x = fmaxf(m.x, s.gscr[j].x);
                    m.y = fmaxf(m.y, s.gscr[j].y);
                }
                s.gmax[it] = m;
            }
        }
        __syncthreads();  // the stages of slots k - 1 and k are read
        issue(k + kClStages - 1);
    }
    cp_async_wait<0>();
    cluster.sync();  // 1: every CTA's screen values and group maxima are complete

    // ---- threshold from every group maximum of the query, then local candidates
    int mode = 0;  // 0: candidates; 1: every eligible chunk kept; 2: exact scan in the leader
    if (ne <= K) mode = 1;
    else if (G < K + 1) mode = 2;
    if (mode == 0) {
        float em = 0.f;
        for (int g = tid; g < G; g += kClThreads) {
            const int owner = g / gper;
            const float2 v = *cluster.map_shared_rank(&s.gmax[g - owner * gper], owner);
            s.gall[g] = v;
            em = fmaxf(em, v.y);
        }
        em = warp_max(em);
        if (lane == 0) s.wmax[warp] = em;
        __syncthreads();
        block_kth_plus_one<kClThreads>(s.gall, G, K, &s.tk);
        __syncthreads();
        if (tid == 0) {
            float e2 = 0.f;
            for (int k = 0; k < kClThreads / 32; ++k) e2 = fmaxf(e2, s.wmax[k]);
            s.cut = __fsub_rd(s.tk, e2);
        }
        __syncthreads();
        const float cut = s.cut;
        for (int lc = tid; lc < nloc; lc += kClThreads) {
            const float2 v = s.scr[lc];
            if (__fadd_ru(v.x, v.y) >= cut) {
                const int pos = atomicAdd(&s.ncand, 1);
                if (pos < kPoolCap) {
                    s.cand.idx[pos] = c_begin + lc;
                    s.cand.s[pos] = v.x;
                    s.cand.e[pos] = v.y;
                }
            }
        }
        __syncthreads();
        // every local candidate is screened again on CUDA cores (the tight radius; four
        // threads each) while its K and V rows are prefetched into L2 for the attend
        // that follows the pick
        const int nc = min(s.ncand, kPoolCap);
        constexpr int kLines = kChunk * D * (int)sizeof(T) / 128;  // 128-byte lines per tile
        for (int l = tid; l < nc * 2 * kLines; l += kClThreads) {
            const int j = l / (2 * kLines), rem = l - j * 2 * kLines, tv = rem / kLines, line = rem - tv * kLines;
            const int row = line * 128 / (D * (int)sizeof(T)), off = line * 128 - row * D * (int)sizeof(T);
            const int64_t pos = (int64_t)s.cand.idx[j] * kChunk + row;
            const uint8_t *p = reinterpret_cast<const uint8_t *>(tv ? vc + pos * aa.V.st : kc + pos * aa.K.st) + off;
            asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
        }
        int tq;
        const QueryCtx q = make_ctx<T, D>(sa, qi, tq);
        rescreen_pool<T, D, kClThreads>(q, s.qs, s.cand, nc);
        __syncthreads();
        // hand the count and the first kPushCap candidates to the leader (remote stores;
        // the next cluster barrier makes them visible there)
        ClSmem<D> &L = *cluster.map_shared_rank(&s, 0);
        for (int j = tid; j < min(nc, kPushCap); j += kClThreads) {
            L.push_idx[rank][j] = s.cand.idx[j];
            L.push_s[rank][j] = s.cand.s[j];
            L.push_e[rank][j] = s.cand.e[j];
        }
        if (tid == 0) L.push_n[rank] = s.ncand;
    }
    cluster.sync();  // 2: every CTA's candidates (and their scores and chunk sums) are complete

    // ---- leader: the exact top-K, written out and published ascending
    if (rank == 0) {
        int tq;
        const QueryCtx q = make_ctx<T, D>(sa, qi, tq);
        if (mode == 0) {
            int total = 0;
            bool fits = true, pushed = true;
            for (int r = 0; r < kCl; ++r) {
                const int n = s.push_n[r];
                fits &= n <= kPoolCap;
                pushed &= n <= kPushCap;
                total += n;
            }
            fits &= total <= kPoolCap;
            if (fits) {
                // the candidates (tight screen values) into the pool, then the exact
                // interval top-K (float64 scores only for the band) in one warp
                int base = 0;
                for (int r = 0; r < kCl; ++r) {
                    const int n = s.push_n[r];
                    // the pushed copies, or (past the push slots) the CTA's own pool
                    const Pool64 &rp = *cluster.map_shared_rank(&s.cand, r);
                    for (int j = tid; j < n; j += kClThreads) {
                        s.pool.idx[base + j] = pushed ? s.push_idx[r][j] : rp.idx[j];
                        s.pool.s[base + j] = pushed ? s.push_s[r][j] : rp.s[j];
                        s.pool.e[base + j] = pushed ? s.push_e[r][j] : rp.e[j];
                        s.pool.x[base + j] = __longlong_as_double(0x7ff8000000000000ll);
                    }
                    base += n;
                }
                __syncthreads();
                if (warp == 0) {
                    Slots<2> sl;
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int j = lane + 32 * r;
                        const bool ok = j < total;
                        sl.idx[r] = ok ? s.pool.idx[j] : -1;
                        sl.s[r] = ok ? s.pool.s[j] : 0.f;
                        sl.e[r] = ok ? s.pool.e[j] : 0.f;
                        sl.x[r] = ok ? s.pool.x[j] : 0.0;
                    }
                    float bnd;
                    const unsigned keep = warp_topk<T, D, 2>(sl, K, q, bnd);
                    __syncwarp();
                    const int n = warp_append<2>(sl, keep, s.out, 0);
                    if (lane == 0) s.out.n = n;
                    __syncwarp();
                    warp_write(s.out, K, qi, sa.idx, sa.score, sa.nsel);
                }
            } else {
                mode = 2;  // more candidates than the lists hold (heavy ties)
            }
        }
        if (mode == 1) {  // every eligible chunk is kept, in index order, with its screen value
            for (int r = tid; r < K; r += kClThreads) {
                float sv = -INFINITY;
                if (r < ne) {
                    const int owner = r / (gper * kGroupRows);
                    sv = cluster.map_shared_rank(s.scr, owner)[r - owner * gper * kGroupRows].x;
                    s.sel_idx[r] = r;
                    s.sel_s[r] = sv;
                }
                sa.idx[qi * K + r] = r < ne ? r : -1;
                sa.score[qi * K + r] = sv;
            }
            if (tid == 0) {
                sa.nsel[qi] = ne;
                s.sel_n = ne;
            }
        } else if (mode == 2 && warp == 0) {  // short table or heavy ties: the exact running-list scan
            warp_scan<T, D>(q, s.qs, 0, ne, K, s.out);
            warp_write(s.out, K, qi, sa.idx, sa.score, sa.nsel);
        }
        if (mode != 1) {
            __syncthreads();
            if (warp == 0) {
                const int n = s.out.n;  // the kept list in ascending chunk index
                if (lane < n) {
                    const int me = s.out.idx[lane];
                    int rk = 0;
                    for (int j = 0; j < n; ++j) rk += s.out.idx[j] < me;
                    s.sel_idx[rk] = me;
                    s.sel_s[rk] = s.out.s[lane];
                }
                if (lane == 0) s.sel_n = n;
            }
        }
        // hand the kept list to every other CTA (remote stores, visible after the barrier)
        __syncthreads();
        for (int r = 1; r < kCl; ++r) {
            ClSmem<D> &R = *cluster.map_shared_rank(&s, r);
            for (int j = tid; j < s.sel_n; j += kClThreads) {
                R.sel_idx[j] = s.sel_idx[j];
                R.sel_s[j] = s.sel_s[j];
            }
            if (tid == 0) R.sel_n = s.sel_n;
        }
    }
    cluster.sync();  // 3: every CTA holds the kept list

    {
        const int nsel = s.sel_n;
        const int *lidx = s.sel_idx;
        const float *lsc = s.sel_s;
        {
            // this CTA's kept chunks (slots rank, rank + 8, ...), two units per round: the
            // K and V tiles of a unit take two stages
            for (int sl0 = rank; sl0 < nsel; sl0 += 2 * kCl) {
                int cu[2];
                float mu[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int sl = sl0 + j * kCl;
                    cu[j] = sl < nsel ? lidx[sl] : -1;
                    mu[j] = sl < nsel ? lsc[sl] : -INFINITY;
                    if (cu[j] >= 0) {
                        const int start = cu[j] * kChunk;
                        tile_issue<T, D>(stage(2 * j), kc + (int64_t)start * aa.K.st, aa.K.st, tile_rows(start));
                        tile_issue<T, D>(stage(2 * j + 1), vc + (int64_t)start * aa.V.st, aa.V.st, tile_rows(start));
                    }
                }
                cp_async_commit();
                cp_async_wait<0>();
                __syncthreads();
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    if (cu[j] < 0) continue;
                    cl_unit<T, D>(s, stage(2 * j), stage(2 * j + 1), tile_rows(cu[j] * kChunk), aa.scale);
                    cl_fold<D>(s, mu[j]);
                }
                __syncthreads();  // the stages are read before the next round refills them
            }
        }
    }
    {  // hand this CTA's running (max, sum, vector) to the leader
        ClSmem<D> &L = *cluster.map_shared_rank(&s, 0);
        for (int x = tid; x < D; x += kClThreads) L.part_acc[rank][x] = s.acc[x];
        if (tid == 0) {
            L.part_m[rank] = s.run_m;
            L.part_z[rank] = s.run_z;
        }
    }
    cluster.sync();  // 4: the leader holds every CTA's partial

    // ---- leader: o = sum_r e^{m_r - M} acc_r / sum_r e^{m_r - M} z_r, lse = M + log(...)
    if (rank == 0) {
        float M = -INFINITY;
        for (int r = 0; r < kCl; ++r) M = fmaxf(M, s.part_m[r]);
        float Z = 0.f;
        for (int r = 0; r < kCl; ++r)
            if (s.part_m[r] != -INFINITY) Z += s.part_z[r] * expf(s.part_m[r] - M);
        T *orow = static_cast<T *>(aa.O.ptr) + b * aa.O.sb + h * aa.O.sh;
        for (int x = tid; x < D; x += kClThreads) {
            float o = 0.f;
            for (int r = 0; r < kCl; ++r)
                if (s.part_m[r] != -INFINITY) o += s.part_acc[r][x] * expf(s.part_m[r] - M);
            orow[x] = (T)(M == -INFINITY ? 0.f : o / Z);
        }
        if (aa.lse && tid == 0) aa.lse[qi] = M == -INFINITY ? -INFINITY : M + logf(Z);
    }
    cluster.sync();  // 5: no CTA leaves while another may still access its shared memory
}

template <typename T, int D>
hils_status launch_cluster(const SelectArgs &sa, const AttendArgs &aa, cudaStream_t st) {
    using Cfg = ClCfg<T, D>;
    constexpr int kSmem = kClStages * Cfg::kStageStride;
    static KernelSetup setup;
    const hils_status stt = kernel_setup(setup, (const void *)decode_cluster_kernel<T, D>, kClThreads, kSmem, nullptr);
    if (stt != HILS_OK) return stt;
    const dim3 grid(kCl, (unsigned)(sa.B * sa.H));
    decode_cluster_kernel<T, D><<<grid, kClThreads, kSmem, st>>>(sa, aa);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace

bool decode_cluster_supported(int B, int H, int C, int K) {
    return (int64_t)B * H >= 16 && (int64_t)B * H <= 65535 && C <= kCl * kClMaxLocal && K >= 1 && K <= kMaxK;
}

hils_status launch_decode_cluster(hils_dtype dt, int d, const SelectArgs &sa, const AttendArgs &aa, cudaStream_t s) {
    if (dt == HILS_BF16) return d == 64 ? launch_cluster<bf16, 64>(sa, aa, s) : launch_cluster<bf16, 128>(sa, aa, s);
    return d == 64 ? launch_cluster<float, 64>(sa, aa, s) : launch_cluster<float, 128>(sa, aa, s);
}

}  // namespace hils
