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
#include "select_common.cuh"

namespace hils {
namespace {

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
// S1 select_screen_kernel: a persistent grid walks (query, 128-row block) items with
// a 3-stage cp.async pipeline; a stage holds the block's summary rows, their biases,
// the query row and the query's position, so no load waits on another. kTPR threads
// share a row (one 16-byte unit each); each thread accumulates its unit's partial dot
// and |k|^2 for kRPT rows with packed float32 FMAs, and a transpose reduction across
// the kTPR lanes leaves each lane the totals of one row. Written to the workspace:
// the screen value s_c and radius e_c of every eligible chunk, and the largest s and
// e of every 64-chunk group. The radius is the Cauchy-Schwarz form of the
// fused-multiply-add dot-product bound, doubled:
//   e_c = scale |q~| |k'_c| (d+2) 2^-23 + |s_c| 2^-22.
// S2 select_pick_kernel (one 1024-thread CTA per query, dependent launch): T = the
// (K+1)-th largest group maximum is attained by K+1 distinct chunks, so the K-th
// largest lo is at least T - e_max and every chunk with hi < T - e_max is certainly
// out. The remaining candidates (typically K + a few) go through the exact interval
// top-K in one warp. With fewer than K+1 groups, T comes from bisection over the
// ordered float keys of the screen values instead. Heavy ties (more than 64
// candidates) fall back to folding the candidates in batches of 32, always exact.

constexpr int kScrThreads = 256;
constexpr int kScrRows = 128;   // summary rows per block (one pipeline stage)
constexpr int kScrStages = 3;
constexpr int kGroupRows = 64;  // rows per group maximum
constexpr int kPickThreads = 1024;
constexpr int kPickItems = 16;  // screen values per pick thread: C <= 16384
constexpr int kPoolCap = 64;
constexpr int kMaxGroups = kPickThreads * kPickItems / kGroupRows;  // 256

template <typename T, int D>
struct ScrCfg {
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kTPR = kRowBytes / 16;            // threads per row: 8, 16 or 32
    static constexpr int kRowGroups = kScrThreads / kTPR;  // rows per step
    static constexpr int kRPT = kScrRows / kRowGroups;     // rows per thread
    static constexpr int kBiasOff = kScrRows * kRowBytes;
    static constexpr int kQOff = kBiasOff + kScrRows * 4;
    static constexpr int kPosOff = kQOff + kRowBytes;
    static constexpr int kStageBytes = kPosOff + 16;
    static constexpr int kSmemBytes = kScrStages * kStageBytes + kScrRows * 8;
    static constexpr int kGroupsPerBlock = kScrRows / kGroupRows;
    static constexpr int kRowGroupsPerGroup = kGroupRows / kRPT;
    static constexpr int kCopies = kScrRows * kTPR / kScrThreads;  // 16-byte copies per thread
    static_assert(2 * kRPT == kTPR, "half-square transpose reduction");
    // bf16 tables are screened on tensor cores (16 rows per warp, swizzled shared rows);
    // float32 tables on CUDA cores (kRPT rows per thread group).
    static constexpr bool kMma = sizeof(T) == 2;
    static constexpr int kSlotRows = kMma ? 16 : kRPT;
    static constexpr int kSlots = kScrRows / kSlotRows;
    static constexpr int kSlotsPerGroup = kGroupRows / kSlotRows;
};

__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ float sqrt_approx(float x) {
    float r;
    asm("sqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Two adjacent elements of a 16-byte vector as a float pair.
__device__ __forceinline__ float2 pair_of(const uint4 &v, int p, bf16) {
    const uint32_t w = p == 0 ? v.x : p == 1 ? v.y : p == 2 ? v.z : v.w;
    return make_float2(bf16lo(w), bf16hi(w));
}
__device__ __forceinline__ float2 pair_of(const uint4 &v, int p, float) {
    return p == 0 ? make_float2(__uint_as_float(v.x), __uint_as_float(v.y))
                  : make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
}

// v[i] holds this lane's partial for row i of its 2N-lane group. Each exchange step
// (lane offset o = N, N/2, ..., 2) sends half of the rows a lane holds to its partner
// and keeps the other half; a last butterfly step adds the pair (l, l^1). Afterwards
// v[0] holds the group total of row (lane_in_group >> 1).
template <int N>
__device__ __forceinline__ void transpose_reduce(float (&v)[N], int lane_in_group) {
#pragma unroll
    for (int o = N; o >= 2; o /= 2) {
        const bool upper = (lane_in_group & o) != 0;
#pragma unroll
        for (int i = 0; i < o / 2; ++i) {
            const float keep = upper ? v[i + o / 2] : v[i];
            const float send = upper ? v[i] : v[i + o / 2];
            v[i] = keep + __shfl_xor_sync(kFull, send, o);
        }
    }
    v[0] += __shfl_xor_sync(kFull, v[0], 1);
}

struct ScreenWs {
    float2 *scr;   // [queries][C]
    float2 *gmax;  // [queries][ceil(C/64)]
};

__host__ __device__ __forceinline__ int groups_of(int C) { return (C + kGroupRows - 1) / kGroupRows; }

__device__ __forceinline__ ScreenWs screen_ws(const SelectArgs &a) {
    const int64_t nq = (int64_t)a.B * a.H * a.Lq;
    ScreenWs w;
    w.scr = reinterpret_cast<float2 *>(static_cast<uint8_t *>(a.ws) + kSelectStatusBytes);
    w.gmax = w.scr + nq * a.C;
    return w;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// Tensor-core screen of one stage (bf16): warp w takes rows 16w..16w+15. Per k-step one
// ldmatrix.x4 of the 16x16 row tile A and three m16n8k16 MMAs: A times q (q in column 0
// of B), and A times its own rows 0-7 and 8-15 (Gram blocks whose diagonals are |k'|^2;
// the B fragments of those are A's own registers). Radius: the tensor-core float32
// accumulation order and rounding are not specified, so the bound allows d * 2^-16 of
// scale |q| |k'| (about 2^7 times the round-to-nearest bound), plus 2^-22 |s| for the
// final fused multiply-add; |k'|^2 itself carries a 2^-8 margin.
template <int D>
__device__ void screen_stage_mma(const uint8_t *st, int q_off, int bias_off, float scale, int c0, int ne,
                                 float2 *scr_row, float2 *slots) {
    constexpr int kRowBytes = D * 2;
    constexpr int kKSteps = D / 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int rbase = warp * 16;
    const uint32_t *qw = reinterpret_cast<const uint32_t *>(st + q_off);
    float qn2 = 0.f;
    for (int pidx = lane; pidx < D / 2; pidx += 32) {
        const uint32_t w = qw[pidx];
        qn2 = fmaf(bf16lo(w), bf16lo(w), fmaf(bf16hi(w), bf16hi(w), qn2));
    }
    qn2 = warp_sum(qn2);
    const int lrow = rbase + (lane & 7) + ((lane >> 3) & 1) * 8;
    const uint32_t row_addr = (uint32_t)__cvta_generic_to_shared(st + lrow * kRowBytes);
    float dacc[4] = {0.f, 0.f, 0.f, 0.f}, g1[4] = {0.f, 0.f, 0.f, 0.f}, g2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < kKSteps; ++ks) {
        uint32_t a[4];
        const int unit = ks * 2 + (lane >> 4);
        ldmatrix_x4(a, row_addr + (uint32_t)((unit ^ (lrow & 7)) * 16));
        const uint32_t b0 = g == 0 ? qw[ks * 8 + tq] : 0u;
        const uint32_t b1 = g == 0 ? qw[ks * 8 + 4 + tq] : 0u;
        mma_bf16_16816(dacc, a, b0, b1);
        mma_bf16_16816(g1, a, a[0], a[2]);
        mma_bf16_16816(g2, a, a[1], a[3]);
    }
    // diagonal of the Gram blocks: row g in lane (g, g>>1), element (g & 1)
    const float d1 = (g & 1) ? g1[1] : g1[0];
    const float d2 = (g & 1) ? g2[3] : g2[2];
    const int src = g * 4 + (g >> 1);
    const float k1 = __shfl_sync(kFull, d1, src);
    const float k2 = __shfl_sync(kFull, d2, src);
    const float *bias = reinterpret_cast<const float *>(st + bias_off);
    const float ecoef = scale * sqrt_approx(qn2) * ((float)D * 0x1p-16f) * (1.f + 0x1p-8f);
    float ms = -INFINITY, me = 0.f;
    if (tq == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = rbase + g + 8 * h;
            const int c = c0 + row;
            const float dot = h ? dacc[2] : dacc[0];
            const float sv = fmaf(dot, scale, bias[row]);
            const float ev = fmaf(ecoef, sqrt_approx(h ? k2 : k1), fabsf(sv) * 0x1p-22f);
            if (c < ne) {
                scr_row[c] = make_float2(sv, ev);
                ms = fmaxf(ms, sv);
                me = fmaxf(me, ev);
            }
        }
    }
    ms = warp_max(ms);
    me = warp_max(me);
    if (lane == 0) slots[warp] = make_float2(ms, me);
}

template <typename T, int D>
__global__ void __launch_bounds__(kScrThreads) select_screen_kernel(SelectArgs a) {
    using Cfg = ScrCfg<T, D>;
    constexpr int kN = Vec<T>::kN;
    extern __shared__ __align__(16) uint8_t smem[];
    float2 *gscr = reinterpret_cast<float2 *>(smem + kScrStages * Cfg::kStageBytes);
    pdl_trigger();
    const int tid = threadIdx.x, col = tid % Cfg::kTPR, rg = tid / Cfg::kTPR;
    const int nblk = (a.C + kScrRows - 1) / kScrRows;
    const int nq = a.B * a.H * a.Lq;
    const ScreenWs ws = screen_ws(a);
    const int G = groups_of(a.C);
    // items (query, block) are walked with a stride of gridDim.x; the (query, block)
    // pair advances by a fixed (q_step, b_step), so no division per item
    const int q_step = (int)(gridDim.x / nblk), b_step = (int)(gridDim.x % nblk);
    struct Item {
        int qi, blk;
    };
    auto advance = [&](Item x) {
        x.blk += b_step;
        x.qi += q_step;
        if (x.blk >= nblk) {
            x.blk -= nblk;
            ++x.qi;
        }
        return x;
    };

    auto issue = [&](Item itm, int stage) {
        if (itm.qi < nq) {
            const int qi = itm.qi, blk = itm.blk;
            const int i = qi % a.Lq;
            const int bh = qi / a.Lq;
            const int h = bh % a.H;
            const int b = bh / a.H;
            const int c0 = blk * kScrRows;
            const int rows = min(kScrRows, a.C - c0);
            uint8_t *st = smem + stage * Cfg::kStageBytes;
            const T *kh = static_cast<const T *>(a.Ksum.ptr) + b * a.Ksum.sb + h * a.Ksum.sh;
            // copy k of this thread: row tid/kTPR + k*(kScrThreads/kTPR), unit tid%kTPR
            const int r0 = tid / Cfg::kTPR;
            const uint8_t *src = reinterpret_cast<const uint8_t *>(kh + (int64_t)(c0 + r0) * a.Ksum.st) + col * 16;
            // bf16 rows are stored with their 16-byte units permuted by (unit ^ (row & 7)), so
            // that the tensor-core fragment loads of 8 rows hit 8 distinct bank groups
            const int dcol = Cfg::kMma ? (col ^ (r0 & 7)) : col;
            uint8_t *dst = st + r0 * Cfg::kRowBytes + dcol * 16;
            const int64_t src_step = (int64_t)(kScrThreads / Cfg::kTPR) * a.Ksum.st * (int64_t)sizeof(T);
#pragma unroll
            for (int k = 0; k < Cfg::kCopies; ++k)
                if (r0 + k * (kScrThreads / Cfg::kTPR) < rows)
                    cp_async16(dst + k * (kScrThreads / Cfg::kTPR) * Cfg::kRowBytes, src + k * src_step);
            const float *brow = a.Bsum + ((int64_t)b * a.H + h) * a.C + c0;
            for (int r = tid; r < rows; r += kScrThreads) cp_async4(st + Cfg::kBiasOff + r * 4, brow + r);
            const T *qrow = static_cast<const T *>(a.Qcal.ptr) + b * a.Qcal.sb + h * a.Qcal.sh + i * a.Qcal.st;
            for (int u = tid; u < Cfg::kTPR; u += kScrThreads)
                cp_async16(st + Cfg::kQOff + u * 16, reinterpret_cast<const uint8_t *>(qrow) + u * 16);
            if (tid == 0) {
                if (a.qpos) cp_async4(st + Cfg::kPosOff, a.qpos + (int64_t)b * a.Lq + i);
                else *reinterpret_cast<int *>(st + Cfg::kPosOff) = i;
            }
        }
        cp_async_commit();
    };

    Item cur{(int)(blockIdx.x / nblk), (int)(blockIdx.x % nblk)};
    Item ahead = cur;
#pragma unroll
    for (int k = 0; k < kScrStages - 1; ++k) {
        issue(ahead, k);
        ahead = advance(ahead);
    }
    int stage = 0;
    for (; cur.qi < nq; cur = advance(cur)) {
        issue(ahead, (stage + kScrStages - 1) % kScrStages);
        ahead = advance(ahead);
        cp_async_wait<kScrStages - 1>();
        __syncthreads();
        const uint8_t *st = smem + stage * Cfg::kStageBytes;
        const int64_t qi = cur.qi;
        const int blk = cur.blk;
        const int c0 = blk * kScrRows;
        const int ne = eligible(*reinterpret_cast<const int *>(st + Cfg::kPosOff), a.C);
        if (c0 < ne && Cfg::kMma) {
            screen_stage_mma<D>(st, Cfg::kQOff, Cfg::kBiasOff, a.scale, c0, ne, ws.scr + qi * a.C, gscr);
        } else if (c0 < ne) {
            // query slice of this thread's unit as float pairs, and |q|^2
            const uint4 qv = *reinterpret_cast<const uint4 *>(st + Cfg::kQOff + col * 16);
            float2 q2[kN / 2];
            float qn2 = 0.f;
#pragma unroll
            for (int p = 0; p < kN / 2; ++p) {
                q2[p] = pair_of(qv, p, T());
                qn2 = fmaf(q2[p].x, q2[p].x, fmaf(q2[p].y, q2[p].y, qn2));
            }
#pragma unroll
            for (int o = Cfg::kTPR / 2; o > 0; o >>= 1) qn2 += __shfl_xor_sync(kFull, qn2, o);
            float dotv[Cfg::kRPT], ksqv[Cfg::kRPT];
#pragma unroll
            for (int r = 0; r < Cfg::kRPT; ++r) {
                const uint4 kv = *reinterpret_cast<const uint4 *>(st + (rg * Cfg::kRPT + r) * Cfg::kRowBytes + col * 16);
                float2 d2 = make_float2(0.f, 0.f), k2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int p = 0; p < kN / 2; ++p) {
                    const float2 kf = pair_of(kv, p, T());
                    d2 = __ffma2_rn(q2[p], kf, d2);
                    k2 = __ffma2_rn(kf, kf, k2);
                }
                dotv[r] = d2.x + d2.y;
                ksqv[r] = k2.x + k2.y;
            }
            transpose_reduce<Cfg::kRPT>(dotv, col);
            transpose_reduce<Cfg::kRPT>(ksqv, col);
            const int row = rg * Cfg::kRPT + (col >> 1);
            const int c = c0 + row;
            const bool valid = c < ne;
            const float ecoef = a.scale * sqrtf(qn2) * ((float)(D + 2) * 0x1p-23f);
            const float sv = fmaf(dotv[0], a.scale, reinterpret_cast<const float *>(st + Cfg::kBiasOff)[row]);
            const float ev = fmaf(ecoef, sqrt_approx(ksqv[0]), fabsf(sv) * 0x1p-22f);
            if (valid && (col & 1) == 0) ws.scr[qi * a.C + c] = make_float2(sv, ev);
            float gs = valid ? sv : -INFINITY, ge = valid ? ev : 0.f;
#pragma unroll
            for (int o = Cfg::kTPR / 2; o > 0; o >>= 1) {
                gs = fmaxf(gs, __shfl_xor_sync(kFull, gs, o));
                ge = fmaxf(ge, __shfl_xor_sync(kFull, ge, o));
            }
            if (col == 0) gscr[rg] = make_float2(gs, ge);
        }
        __syncthreads();
        if (c0 < ne && tid < Cfg::kGroupsPerBlock) {
            const int g0 = tid * Cfg::kSlotsPerGroup;
            float2 m = gscr[g0];
            for (int k = 1; k < Cfg::kSlotsPerGroup; ++k) {
                m.x = fmaxf(m.x, gscr[g0 + k].x);
                m.y = fmaxf(m.y, gscr[g0 + k].y);
            }
            const int g = blk * Cfg::kGroupsPerBlock + tid;
            if (g * kGroupRows < ne) ws.gmax[qi * G + g] = m;
        }
        __syncthreads();
        stage = (stage + 1) % kScrStages;
    }
    cp_async_wait<0>();
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

// (K+1)-th largest of n <= 256 values in shared memory (one warp; duplicates counted).
__device__ float warp_kth_plus_one(const float2 *v, int n, int K) {
    const int lane = threadIdx.x & 31;
    unsigned keys[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int g = lane + 32 * r;
        keys[r] = g < n ? ordered_key(v[g].x) : 0u;
    }
    unsigned taken = 0, wmax = 0;
    for (int it = 0; it <= K; ++it) {
        unsigned best = 0u;
        int bslot = -1;
#pragma unroll
        for (int r = 0; r < 8; ++r)
            if (!(taken >> r & 1) && keys[r] > best) {
                best = keys[r];
                bslot = r;
            }
        wmax = __reduce_max_sync(kFull, best);
        const unsigned owners = __ballot_sync(kFull, bslot >= 0 && best == wmax);
        if (lane == __ffs(owners) - 1) taken |= 1u << bslot;
    }
    return key_to_float(wmax);
}

template <typename T, int D>
__global__ void __launch_bounds__(kPickThreads) select_pick_kernel(SelectArgs a) {
    __shared__ float fscr[32];
    __shared__ int iscr[32];
    __shared__ Pool64 pool;
    __shared__ EntryList out;
    __shared__ float2 gm[kMaxGroups];
    __shared__ float thr[2];
    __shared__ __align__(16) float qs[D];
    pdl_wait();     // the screen grid has completed and its writes are visible
    pdl_trigger();  // let the next dependent-launched kernel be scheduled
    const int64_t qi = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    int t;
    const QueryCtx q = make_ctx<T, D>(a, qi, t);
    if (tid < D) qs[tid] = (float)static_cast<const T *>(q.qrow)[tid];
    const int ne = eligible(t, a.C);
    const int K = a.topk;
    const ScreenWs ws = screen_ws(a);
    const float2 *scr = ws.scr + qi * a.C;
    if (ne <= K) {  // every eligible chunk is kept, in index order
        for (int r = tid; r < K; r += kPickThreads) {
            a.idx[qi * K + r] = r < ne ? r : -1;
            a.score[qi * K + r] = r < ne ? __ldcg(&scr[r]).x : -INFINITY;
        }
        if (tid == 0) a.nsel[qi] = ne;
        return;
    }
    const int G = groups_of(ne);
    float sv[kPickItems], ev[kPickItems];
#pragma unroll
    for (int j = 0; j < kPickItems; ++j) {
        const int c = tid + j * kPickThreads;
        const float2 v = c < ne ? __ldcg(&scr[c]) : make_float2(-INFINITY, 0.f);
        sv[j] = v.x;
        ev[j] = v.y;
    }
    float thresh = 0.f, emax = 0.f;
    int total = 0, wbase = 0, incl = 0, mine = 0;
    // Candidate count above cut = T - e_max, and this thread's offset in the pool.
    auto count_candidates = [&](float thr_value) {
        const float cut = __fsub_rd(thr_value, emax);
        mine = 0;
#pragma unroll
        for (int j = 0; j < kPickItems; ++j) mine += sv[j] != -INFINITY && __fadd_ru(sv[j], ev[j]) >= cut;
        incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += v;
        }
        __syncthreads();
        if (lane == 31) iscr[w] = incl;
        __syncthreads();
        wbase = 0;
        for (int k = 0; k < w; ++k) wbase += iscr[k];
        total = 0;
        for (int k = 0; k < kPickThreads / 32; ++k) total += iscr[k];
    };
    bool have = false;
    if (G >= K + 1) {
        // T = (K+1)-th largest maximum of the 64-chunk groups; e_max = largest group radius
        const float2 *gmx = ws.gmax + qi * groups_of(a.C);
        for (int g = tid; g < G; g += kPickThreads) gm[g] = __ldcg(&gmx[g]);
        __syncthreads();
        if (w == 0) {
            float em = 0.f;
            for (int g = lane; g < G; g += 32) em = fmaxf(em, gm[g].y);
            em = warp_max(em);
            const float tk = warp_kth_plus_one(gm, G, K);
            if (lane == 0) {
                thr[0] = tk;
                thr[1] = em;
            }
        }
        __syncthreads();
        thresh = thr[0];
        emax = thr[1];
        count_candidates(thresh);
        have = total <= kPoolCap;
    }
    if (!have) {
        // few groups: bisection over the ordered keys of the screen values, with the
        // invariant count(>= lo_key) >= K+1 and count(>= hi_key) <= K
        float em = 0.f, smax = -INFINITY, smin = INFINITY, sum = 0.f, sum2 = 0.f;
#pragma unroll
        for (int j = 0; j < kPickItems; ++j) {
            if (sv[j] != -INFINITY) {
                em = fmaxf(em, ev[j]);
                smax = fmaxf(smax, sv[j]);
                smin = fminf(smin, sv[j]);
                sum += sv[j];
                sum2 = fmaf(sv[j], sv[j], sum2);
            }
        }
        emax = block_reduce_f<1>(em, fscr);
        smax = block_reduce_f<1>(smax, fscr);
        smin = block_reduce_f<2>(smin, fscr);
        sum = block_reduce_f<0>(sum, fscr);
        sum2 = block_reduce_f<0>(sum2, fscr);
        unsigned lo_key = ordered_key(smin), hi_key = ordered_key(smax) + 1u;
        const float mu = sum / ne;
        const float sd = sqrtf(fmaxf(sum2 / ne - mu * mu, 0.f));
        const float p = fminf((float)(K + 8) / (float)ne, 0.49f);
        unsigned tk = min(max(ordered_key(mu + normal_upper_quantile(p) * sd), lo_key), hi_key - 1u);
        for (int it = 0; it < 40; ++it) {
            int cnt = 0;
#pragma unroll
            for (int j = 0; j < kPickItems; ++j) cnt += sv[j] != -INFINITY && ordered_key(sv[j]) >= tk;
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
        thresh = key_to_float(tk);
        count_candidates(thresh);
    }
    const float cut = __fsub_rd(thresh, emax);
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
        __syncthreads();  // every candidate is in the pool before any thread reads it
        // the candidates are screened again on CUDA cores (round-to-nearest fused
        // multiply-adds: the tight radius), so that few need the float64 score
        if (w < 2 && tid < total) {
            const int c = pool.idx[tid];
            if (c >= 0 && c < ne) screen<T, D>(q, qs, c, pool.s[tid], pool.e[tid]);
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
    if (a.path == kSelectTc) return launch_select_tc(a, s);
    if (a.path == kSelectWarp) {
        const int64_t grid = (nq + kWarps - 1) / kWarps;
        select_warp_kernel<T, D><<<(unsigned)grid, kThreads, 0, s>>>(a);
    } else {
        using Cfg = ScrCfg<T, D>;
        static KernelSetup setup;
        int per_sm = 1;
        hils_status st = kernel_setup(setup, (const void *)select_screen_kernel<T, D>, kScrThreads,
                                      Cfg::kSmemBytes, &per_sm);
        if (st != HILS_OK) return st;
        const int64_t items = nq * ((a.C + kScrRows - 1) / kScrRows);
        const int64_t slots = (int64_t)per_sm * device_sm_count();
        select_screen_kernel<T, D><<<(unsigned)(items < slots ? items : slots), kScrThreads, Cfg::kSmemBytes, s>>>(a);
        st = record_cuda_error(cudaGetLastError());
        if (st != HILS_OK) return st;
        return launch_dependent((const void *)select_pick_kernel<T, D>, dim3((unsigned)nq), dim3(kPickThreads),
                                0, s, a);
    }
    return record_cuda_error(cudaGetLastError());
}

}  // namespace

void select_plan(hils_dtype dt, int d, int B, int H, int Lq, int C, int K, bool has_qpos, int num_sms,
                 SelectArgs *a) {
    const int64_t nq = (int64_t)B * H * Lq;
    a->tiles_per_warp = (C + kTile - 1) / kTile;
    a->ctas_per_query = 0;
    // many queries: tensor-core scoring when the shape allows, else one warp per
    // query; short tables or tables beyond the pick kernel's register capacity also
    // take the warp kernel; otherwise screen + pick
    if (nq >= (int64_t)kWarps * num_sms || C <= kTile || C > kPickThreads * kPickItems || nq > 65535) {
        a->path = select_tc_supported(dt, d, B, H, Lq, C, K, has_qpos) && nq >= (int64_t)kWarps * num_sms
                      ? kSelectTc
                      : kSelectWarp;
        return;
    }
    a->path = kSelectSplit;
    a->ctas_per_query = (C + kScrRows - 1) / kScrRows;
}

size_t select_ws_bytes(int queries, int C, int path) {
    if (path != kSelectSplit) return kSelectStatusBytes;
    // screen value and radius per (query, chunk), then the group maxima per query
    return kSelectStatusBytes + (size_t)queries * (C + groups_of(C)) * sizeof(float2);
}

hils_status launch_select(hils_dtype dt, int d, const SelectArgs &a, cudaStream_t s) {
    if (dt == HILS_BF16) return d == 64 ? launch<bf16, 64>(a, s) : launch<bf16, 128>(a, s);
    return d == 64 ? launch<float, 64>(a, s) : launch<float, 128>(a, s);
}

}  // namespace hils
