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
#include "screen_stage.cuh"

namespace hils {
namespace {

// Groups of G > 1 heads: one warp per (b, group, query) scores every chunk for all of the
// group's heads (their query rows in shared memory as float32) and keeps the exact top K
// of the heads' maximum.
template <typename T, int D>
__global__ void __launch_bounds__(kWarpKernelThreads) select_group_kernel(SelectArgs a) {
    __shared__ __align__(16) float qs_all[kWarpKernelWarps][kMaxGroup * D];
    __shared__ EntryList lists[kWarpKernelWarps];
    const int w = threadIdx.x >> 5;
    const int64_t qg = (int64_t)blockIdx.x * kWarpKernelWarps + w;
    if (qg >= (int64_t)a.B * (a.H / a.G) * a.Lq) return;
    int t, b, g, i;
    const GroupCtx q = make_group_ctx<T, D>(a, qg, t, b, g, i);
    const int ne = eligible(t, a.C, a.excl_w);
    for (int hh = 0; hh < q.G; ++hh) load_query_f32<T, D>(head_ctx(q, hh, (int)sizeof(T)), qs_all[w] + hh * D);
    __syncwarp();
    warp_scan<T, D>(q, qs_all[w], 0, ne, a.topk, lists[w]);
    group_write<T, D>(q, qs_all[w], lists[w], a, qg, b, g, i);
}

// Many queries: one warp per query, direct output.
template <typename T, int D>
__global__ void __launch_bounds__(kWarpKernelThreads) select_warp_kernel(SelectArgs a) {
    __shared__ __align__(16) float qs_all[kWarpKernelWarps][D];
    __shared__ EntryList lists[kWarpKernelWarps];
    const int w = threadIdx.x >> 5;
    const int64_t qi = (int64_t)blockIdx.x * kWarpKernelWarps + w;
    const int64_t nq = (int64_t)a.B * a.H * a.Lq;
    if (qi >= nq) return;
    int t;
    const QueryCtx q = make_ctx<T, D>(a, qi, t);
    const int ne = eligible(t, a.C, a.excl_w);
    load_query_f32<T, D>(q, qs_all[w]);
    __syncwarp();
    warp_scan<T, D>(q, qs_all[w], 0, ne, a.topk, lists[w]);
    warp_write(lists[w], a.topk, qi, a.idx, a.score, a.nsel);
}

// ---- decode-shaped search (few queries, long contexts): screen, then pick
//
// select_screen_kernel: a persistent grid of 256-thread CTAs (2 per SM) walks the
// (query, 128-row block) items, query-major, with a stride of the grid size, through a
// 3-stage ring; a stage holds the block's summary rows (bf16: one TMA tile load per
// 64-column block, completing on the stage's mbarrier; float32: cp.async), their
// biases, the query row and the query's position (cp.async), so no load waits on
// another. Every mbarrier wait is bounded: on expiry the CTA sets the select's status
// word, stops, and lets its copies in flight land before it exits. Rows of either type
// are screened on CUDA cores (kTPR threads per row, packed float32 FMAs, a transpose
// reduction; |k'|^2 from the same loads). Written to the workspace: the screen value s_c
// and radius e_c of every eligible chunk and the largest s and e of every 64-chunk
// group. For grouped
// heads an item is a (b, group, query) and its block of the G heads' tables, screened
// head after head by the same CTA; each head's interval s_c +- e_c is folded into the
// group's [max lo, max hi] in shared memory, and the group's centre and radius are
// written once, so the pick reads one row per group as for one head.
//   e_c = scale |q~| |k'_c| (d+2) 2^-23 + |s_c| 2^-22 (Cauchy-Schwarz form of the
//   fused-multiply-add bound, doubled).
// select_pick_kernel (one 256-thread CTA per query, dependent launch): T = the (K+1)-th
// largest group maximum is attained by K+1 distinct chunks, so the K-th largest lo is
// at least T - e_max and every chunk with hi < T - e_max is certainly out. Only the
// groups whose max s + max e reaches that cut are read again; their candidates
// (typically K + a few) go through the exact interval top-K in one warp with their
// screen values and radii; for grouped heads (one CTA per (b,
// group, query)) every candidate gets each head's float64 score instead, one thread per
// (head, candidate), and a parallel rank of the group maxima keeps the top K. With fewer
// than K+1 groups the exact running-list scan runs over every chunk instead. Heavy ties
// (more than 64 candidates) fall back to folding the candidates in batches of 32, always
// exact. The (K+1)-th group maximum is found by a parallel rank count over at most 256
// values.

constexpr int kScrThreads = 256;
constexpr int kPickThreads = 256;
constexpr int kScrRows = 128;   // summary rows per item (one pipeline stage)
constexpr int kDecStages = 3;   // pipeline stages (2 CTAs per SM for bf16 rows of d = 128)

template <typename T, int D>
struct ScrCfg : StageCfg<T, D, kScrThreads, kScrRows> {
    using Base = StageCfg<T, D, kScrThreads, kScrRows>;
    static constexpr int kStages = Base::kStageBytes > 40000 ? 2 : kDecStages;
    static constexpr int kGscrOff = kStages * Base::kStageBytes;
    static constexpr int kFoldOff = kGscrOff + kScrRows * 8;  // grouped heads: one head's (s, e), the group's (lo, hi)
    static constexpr int kSmemBytes = kFoldOff + 2 * kScrRows * 8 + (Base::kTma ? 1024 : 0);  // + alignment slack
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};
// One CTA per query (per (b, group, query) for grouped heads), dependent-launched after
// the screen grid.
template <typename T, int D, bool kGroup>
__global__ void __launch_bounds__(kPickThreads) select_pick_kernel(SelectArgs a) {
    __shared__ PickSmem ps;
    pdl_wait();     // the screen grid has completed and its writes are visible
    pdl_trigger();  // let the next dependent-launched kernel be scheduled
    pick_unit<T, D, kPickThreads, kGroup>(a, screen_ws(a), blockIdx.x, ps);
}

template <typename T, int D, bool kFold>
__global__ void __launch_bounds__(kScrThreads) select_screen_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                    SelectArgs a) {
    using Cfg = ScrCfg<T, D>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // bf16 stages: 1024-byte alignment by pointer arithmetic on the shared array
    uint8_t *smem = Cfg::kTma ? smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u) : smem_raw;
    __shared__ unsigned long long sbar[kDecStages];
    __shared__ uint32_t sabort;
    float2 *gscr = reinterpret_cast<float2 *>(smem + Cfg::kGscrOff);
    // dependent launch: this grid may be scheduled while the preceding kernel drains, so
    // it waits for that kernel (and its memory) before touching anything; then it lets the
    // pick be scheduled
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x;
    if (tid == 0) {
        sabort = 0u;
        if (Cfg::kTma) {
            for (int k = 0; k < Cfg::kStages; ++k) tc::mbar_init(tc::smem_u32(&sbar[k]), 1);
            asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        }
    }
    __syncthreads();
    int tma_issued[kDecStages] = {0, 0, 0};  // thread 0: row loads started per stage
    const int nblk = (a.C + kScrRows - 1) / kScrRows;
    const int gh = kFold ? a.G : 1;           // heads folded per item (1: one query head)
    const int nu = a.B * (a.H / gh) * a.Lq;   // query units: queries, or (b, group, query)
    const int total = nu * nblk;  // checked on the host to fit in int
    const ScreenWs ws = screen_ws(a);
    const int G = groups_of(a.C);
    float2 *tmp = reinterpret_cast<float2 *>(smem + Cfg::kFoldOff);  // one head's (s, e) per row
    float2 *lohi = tmp + kScrRows;                                    // the group's (lo, hi) per row
    // items are unit-major (item = unit * nblk + block), walked with a stride of
    // gridDim.x; each item is gh stages, one per head, in turn
    const int first = blockIdx.x, stride = gridDim.x;
    auto item_of_seq = [&](int sq) { return first + (sq / gh) * stride; };
    // every thread issues its share of the copies of stage sequence number sq into stage `stage`
    auto issue = [&](int sq, int stage) {
        const int item = item_of_seq(sq);
        if (item < total) {
            const int qu = item / nblk, blk = item - (item / nblk) * nblk;
            const int i = qu % a.Lq;
            const int bu = qu / a.Lq;
            const int h = (bu % (a.H / gh)) * gh + sq % gh;
            const int b = bu / (a.H / gh);
            const int c0 = blk * kScrRows;
            const T *kh = static_cast<const T *>(a.Ksum.ptr) + b * a.Ksum.sb + h * a.Ksum.sh;
            const T *qrow = static_cast<const T *>(a.Qcal.ptr) + b * a.Qcal.sb + h * a.Qcal.sh + i * a.Qcal.st;
            stage_issue<T, Cfg>(smem + stage * Cfg::kStageBytes, kh, a.Ksum.st, c0, min(kScrRows, a.C - c0),
                                a.Bsum + ((int64_t)b * a.H + h) * a.C + c0, qrow,
                                a.qpos ? a.qpos + (int64_t)b * a.Lq + i : nullptr, i);
            if (Cfg::kTma && tid == 0) {  // the rows: (D / 64) boxes of 128 rows x 64 columns
                const uint32_t bar = tc::smem_u32(&sbar[stage]);
                const uint32_t dst = tc::smem_u32(smem + stage * Cfg::kStageBytes);
                ++tma_issued[stage];
                tc::mbar_expect_tx(bar, kScrRows * D * 2);
#pragma unroll
                for (int x = 0; x < D / 64; ++x) tc::tma_load_4d(dst + x * kScrRows * 128, &tmK, bar, x * 64, c0, h, b);
            }
        }
        cp_async_commit();
    };

    for (int k = 0; k < Cfg::kStages - 1; ++k) issue(k, k);
    int stage = 0;
    for (int sq = 0; item_of_seq(sq) < total; ++sq) {
        const int item = item_of_seq(sq), hh = sq % gh;
        issue(sq + Cfg::kStages - 1, (stage + Cfg::kStages - 1) % Cfg::kStages);
        cp_async_wait<Cfg::kStages - 1>();
        if (Cfg::kTma) {  // the stage's rows: use sq / kStages of its barrier
            const uint32_t bar = tc::smem_u32(&sbar[stage]), par = (uint32_t)(sq / Cfg::kStages) & 1u;
            bool ok = tc::mbar_try_wait(bar, par);
            const uint64_t t0 = global_ns();
            for (int it = 0; !ok; ++it) {
                ok = tc::mbar_try_wait(bar, par);
                if (!ok && (it & 15) == 15 && (long long)(global_ns() - t0) > a.wait_ns) break;
            }
            if (!ok) {
                sabort = 1u;
                atomicOr(static_cast<uint32_t *>(a.ws), 1u);
            }
        }
        __syncthreads();
        if (Cfg::kTma && sabort) break;  // uniform: read after the barrier
        const uint8_t *st = smem + stage * Cfg::kStageBytes;
        const int qu = item / nblk, blk = item - (item / nblk) * nblk;
        const int c0 = blk * kScrRows;
        const int ne = eligible(*reinterpret_cast<const int *>(st + Cfg::kPosOff) + a.qpos_bias, a.C, a.excl_w);
        float2 *out = kFold ? tmp : ws.scr + (int64_t)qu * a.C;
        const int base = kFold ? c0 : 0;
        if (c0 < ne) {
            screen_stage_fma<T, D, Cfg>(st, a.scale, c0, ne, out, base, gscr);
        }
        __syncthreads();
        if (kFold && c0 < ne) {
            // fold this head's intervals into the group's; after the last head write the
            // group's centre and radius, and its 64-chunk maxima through the slots
            const bool last = hh == gh - 1;
            for (int r = tid; r < kScrRows; r += kScrThreads) {
                const int c = c0 + r;
                float s = -INFINITY, e = 0.f;
                if (c < ne) {
                    const float2 v = tmp[r];
                    float lo = __fsub_rd(v.x, v.y), hi = __fadd_ru(v.x, v.y);
                    if (hh > 0) {
                        lo = fmaxf(lo, lohi[r].x);
                        hi = fmaxf(hi, lohi[r].y);
                    }
                    lohi[r] = make_float2(lo, hi);
                    if (last) {
                        interval_mid(lo, hi, s, e);
                        ws.scr[(int64_t)qu * a.C + c] = make_float2(s, e);
                    }
                }
                if (last) {  // 32-row slot maxima (kScrRows = 128 rows, one warp-row each)
                    const float ms = warp_max(s), me = warp_max(e);
                    if ((tid & 31) == 0) gscr[r >> 5] = make_float2(ms, me);
                }
            }
            __syncthreads();
            if (last && tid < Cfg::kGroupsPerBlock) {
                float2 m = gscr[2 * tid];
                m.x = fmaxf(m.x, gscr[2 * tid + 1].x);
                m.y = fmaxf(m.y, gscr[2 * tid + 1].y);
                const int g = blk * Cfg::kGroupsPerBlock + tid;
                if (g * kGroupRows < ne) ws.gmax[(int64_t)qu * G + g] = m;
            }
        } else if (c0 < ne && tid < Cfg::kGroupsPerBlock) {
            const int g0 = tid * Cfg::kSlotsPerGroup;
            float2 m = gscr[g0];
            for (int k = 1; k < Cfg::kSlotsPerGroup; ++k) {
                m.x = fmaxf(m.x, gscr[g0 + k].x);
                m.y = fmaxf(m.y, gscr[g0 + k].y);
            }
            const int g = blk * Cfg::kGroupsPerBlock + tid;
            if (g * kGroupRows < ne) ws.gmax[(int64_t)qu * G + g] = m;
        }
        __syncthreads();
        stage = (stage + 1) % Cfg::kStages;
    }
    cp_async_wait<0>();
    if (Cfg::kTma && tid == 0) {
        // after an abort: every row load started lands before the CTA releases its memory
        // (each was issued after the previous use of its stage had completed)
        for (int k = 0; k < Cfg::kStages; ++k) {
            if (tma_issued[k] == 0) continue;
            const uint32_t bar = tc::smem_u32(&sbar[k]), par = (uint32_t)(tma_issued[k] - 1) & 1u;
            const uint64_t t0 = global_ns();
            while (!tc::mbar_try_wait(bar, par))
                if ((long long)(global_ns() - t0) > kDrainLimitNs) break;
        }
    }
}

template <typename T, int D>
hils_status launch_screen(const SelectArgs &a, cudaStream_t s) {
    using Cfg = ScrCfg<T, D>;
    static KernelSetup setup1, setupg;
    const void *fn = a.G > 1 ? (const void *)select_screen_kernel<T, D, true> : (const void *)select_screen_kernel<T, D, false>;
    int per_sm = 1;
    const hils_status st = kernel_setup(a.G > 1 ? setupg : setup1, fn, kScrThreads, Cfg::kSmemBytes, &per_sm);
    if (st != HILS_OK) return st;
    const int64_t nu = (int64_t)a.B * (a.H / a.G) * a.Lq;
    const int64_t items = nu * ((a.C + kScrRows - 1) / kScrRows);
    const int64_t slots = (int64_t)per_sm * device_sm_count();
    const int64_t grid = items < slots ? items : slots;
    CUtensorMap mk{};  // bf16 rows come by TMA; float32 rows do not use the map
    if (Cfg::kTma && !tc::make_map(&mk, View{a.Ksum.ptr, a.Ksum.sb, a.Ksum.sh, a.Ksum.st}, a.B, a.H, a.C, kScrRows, D))
        return HILS_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kScrThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    SelectArgs args = a;
    void *argv[] = {&mk, &args};
    return record_cuda_error(cudaLaunchKernelExC(&cfg, fn, argv));
}

template <typename T, int D>
hils_status launch(const SelectArgs &a, cudaStream_t s) {
    const int64_t nq = (int64_t)a.B * a.H * a.Lq;
    if (nq == 0) return HILS_OK;
    if (a.path == kSelectTc) return launch_select_tc(a, s);
    if (a.path == kSelectGroup) {
        const int64_t ng = (int64_t)a.B * (a.H / a.G) * a.Lq;
        select_group_kernel<T, D><<<(unsigned)((ng + kWarpKernelWarps - 1) / kWarpKernelWarps), kWarpKernelThreads, 0,
                                    s>>>(a);
    } else if (a.path == kSelectWarp) {
        const int64_t grid = (nq + kWarpKernelWarps - 1) / kWarpKernelWarps;
        select_warp_kernel<T, D><<<(unsigned)grid, kWarpKernelThreads, 0, s>>>(a);
    } else {
        const hils_status st = launch_screen<T, D>(a, s);
        if (st != HILS_OK) return st;
        if (a.G > 1)
            return launch_dependent((const void *)select_pick_kernel<T, D, true>, dim3((unsigned)(nq / a.G)),
                                    dim3(kPickThreads), 0, s, a);
        return launch_dependent((const void *)select_pick_kernel<T, D, false>, dim3((unsigned)nq),
                                dim3(kPickThreads), 0, s, a);
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
    // query (per (b, group, query) for grouped heads); short tables or tables beyond
    // the pick kernel's register capacity also take the warp kernel; otherwise
    // screen + pick
    if (nq >= (int64_t)kWarpKernelWarps * num_sms || C <= kTile || C > kMaxDecC || nq > 65535 || K < 1) {
        a->path = select_tc_supported(dt, d, B, H, Lq, C, K, has_qpos, a->G) &&
                          nq >= (int64_t)kWarpKernelWarps * num_sms
                      ? kSelectTc
                  : a->G > 1 ? kSelectGroup
                             : kSelectWarp;
        return;
    }
    a->path = kSelectSplit;
    a->ctas_per_query = 1;
}

size_t select_ws_bytes(int queries, int C, int path) {
    if (path != kSelectSplit) return kSelectStatusBytes;
    // screen value and radius per (query, chunk), then the group maxima per query
    return dec_ws_bytes(queries, C);
}

hils_status launch_select(hils_dtype dt, int d, const SelectArgs &a, cudaStream_t s) {
    if (dt == HILS_BF16) return d == 64 ? launch<bf16, 64>(a, s) : launch<bf16, 128>(a, s);
    return d == 64 ? launch<float, 64>(a, s) : launch<float, 128>(a, s);
}

}  // namespace hils
