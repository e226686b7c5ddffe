// Attend backward on the 5th-generation tensor cores (bf16, d = 128): the key-major walk
// of the hierarchical softmax's gradient ("Hierarchical Sparse Attention Done Right"
// (picx.dev summary), Methodology 2, Eq. 10, differentiated by hand; the formulas are
// listed at the top of backward.cu).
//
// A work item is a 64-key block of one (b, h), either a kept chunk with a run of at most
// 1024 of the queries that kept it (entries of the group's inverted index), or a block of
// window keys with a run of at most 1024 of the consecutive queries whose window reaches
// it, walked 128 queries per step. One persistent CTA per SM takes the items in turn (its
// stride over the item list), its pipelines running on across items. With Q and dO the
// step's 128 query rows and K, V the block's 64 keys:
//   S = Q K^T, T = dO V^T            tcgen05, M = 128 queries, N = 64 keys, K = 128 dims
//   per query row (its TMEM lane, two threads with half of the keys each): the
//     softmax-backward weights of the row, dl = scale * weights and cv, both rounded to
//     bf16 into shared memory, and for a kept chunk the score gradient dscore
//   dK^T += Q^T dl, dV^T += dO^T cv  tcgen05, M = 128 dims, N = 64 keys, K = 128 queries
//                                    (Q, dO and dl, cv read as MN-major operands)
//   dQ = dl K                        tcgen05, M = 128 queries, N = 128 dims, K = 64 keys
// Each step's dQ rows are added to the float32 dQ with vector atomic adds; dK^T and dV^T
// stay in TMEM for the whole item and are added to dK and dV once at its end.
// Warp roles (352 threads), all hand-offs through mbarriers:
//   warps 0-7  softmax rows and the dQ, dK, dV epilogues: warp w takes the rows of TMEM
//              lane quadrant w % 4 and half w / 4 of the keys (and of dQ's columns); the
//              two halves of a row exchange its max and sums through shared memory;
//   warps 8-9  loads, into a ring of two stages: the block's K and V (TMA tiles), each
//              step's rows of Q (warp 8) and of dO (warp 9) from the contiguous bf16
//              copies (a chunk's scattered queries: TMA row gathers, four rows per copy;
//              a window block's consecutive queries: one 128-row TMA tile per 64-column
//              half), and the rows' scalars (warp 8), loaded a step ahead;
//   warp 10    allocates TMEM and issues tcgen05.mma (one lane), each product as soon as
//              its inputs are ready.
// S and T are double-buffered in TMEM, so that the products of step s+1 run while the
// softmax of step s does. TMEM columns: S, T of buffer 0 [0, 128), of buffer 1
// [128, 256), dK^T [256, 320), dV^T [320, 384), dQ [384, 512).
// Every mbarrier wait is bounded in time (the global timer): on expiry the CTA sets bit 0
// of the call's status word, every role stops, the copies and MMAs already started are
// awaited (bounded again), TMEM is freed and the CTA exits without its remaining
// gradient adds.
#include <algorithm>

#include "backward_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

using namespace tc;

constexpr int kQ = 128;      // queries per step (TMEM lanes)
constexpr int kKeys = 64;    // keys per block
constexpr int kDim = 128;    // head dimension
constexpr int kThr = 352;
constexpr int kLoadWarp = 8, kMmaWarp = 10;  // load warps 8 (Q, scalars) and 9 (dO)
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// shared memory map (offsets from the 1024-aligned base); every operand region holds
// 128-byte rows with the 128-byte swizzle (16-byte unit u of row r at r * 128 +
// ((u ^ (r % 8)) * 16)), 64-column halves of a 128-column row in separate regions
constexpr int kKOff = 0;                 // K block: 2 halves x [64 keys x 128 B]
constexpr int kVOff = 16384;             // V block, same
constexpr int kQOff = 32768;             // 2 stages x 2 halves x [128 rows x 128 B]
constexpr int kDOOff = kQOff + 65536;    // dO rows, same
constexpr int kDLOff = kDOOff + 65536;   // dl [128 queries x 64 keys] bf16
constexpr int kCVOff = kDLOff + 16384;   // cv, same
constexpr int kScOff = kCVOff + 16384;   // 2 stages x [128] row scalars (int4)
constexpr int kXOff = kScOff + 4096;    // softmax half-row exchange: [2][128] max, [2][128] (sum, o.dO)
constexpr int kBarOff = kXOff + 3072;    // mbarriers
constexpr int kMiscOff = kBarOff + 256;  // TMEM base, abort flag
constexpr int kSmemBytes = kMiscOff + 64 + 1024;  // + alignment slack

enum {
    kBarFull = 0,     // + stage: Q, dO rows (bytes) and scalars (32 arrivals of warp 8) of a step landed
    kBarEmpty = 2,    // + stage: every MMA that read the stage completed
    kBarKV = 4,       // K and V of the item's block landed
    kBarStFull = 5,   // + buffer: S, T written
    kBarStFree = 7,   // + buffer: the softmax warps read S, T (8 arrivals)
    kBarDlFull = 9,   // dl, cv of the step written (8 arrivals)
    kBarDqFull = 10,  // dQ of the step (and every earlier MMA) completed
    kBarDqFree = 11,  // the softmax warps read dQ (8 arrivals)
    kBarDone = 12,    // every MMA of the item completed: dK^T, dV^T final, K and V free
    kBarDrain = 13,   // the MMA warp's own drain
    kBarPair = 14,    // + 2 quadrant + round: the two warps of a row quadrant exchanged half-row
                      //   maxima (round 0) or sums (round 1) (64 arrivals)
    kBarDkvFree = 22, // the softmax warps read the item's dK^T, dV^T (8 arrivals)
    kNumBars = 23
};

// Four rows (y0..y3) of 64 bf16 at column x of a 2-D tensor map into 512 consecutive
// bytes of shared memory (128-byte swizzle, rows in order).
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y0,
                                            int y1, int y2, int y3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4, %5, %6, %7}], [%2];\n" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
        : "memory");
}

// A (64 elements x 128 rows) tile at column x, row y of a 2-D tensor map (128-byte swizzle).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];\n" ::"r"(
            dst),
        "l"(map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// One work item of the walk (uniform over the CTA): item j of the flattened grid of
// (item slot x, (b, h)) pairs; slots beyond a group's chunk-item count, and empty runs,
// are not valid.
struct BwdItem {
    bool valid, chunk;
    int b, h, hk, bh, j0, rows, qb, qe, ns;
};

__device__ __forceinline__ BwdItem decode_item(const BwdTcArgs &t, int j, int gx) {
    const BwdAttendArgs &a = t.a;
    BwdItem it;
    const int x = j % gx;
    it.bh = j / gx;
    it.b = it.bh / a.H;
    it.h = it.bh % a.H;
    const int Hk = a.H / a.G;
    it.hk = it.h / a.G;
    int blk;
    it.valid = true;
    if (x < t.nwin) {
        blk = x / t.nsegw;
        const int seg = x - blk * t.nsegw;
        const int jb = blk * kKeys, nk = min(kKeys, a.N - jb);
        const int qend = min(a.N, jb + nk - 1 + a.W);  // queries whose window reaches the block
        it.qb = jb + seg * kBwdItemQueries;
        it.qe = min(qend, it.qb + kBwdItemQueries);
        it.chunk = false;
    } else {
        const int ci = x - t.nwin;
        const int64_t bg = (int64_t)it.b * Hk + it.hk;
        it.chunk = true;
        if (ci >= t.nitems[bg]) {
            it.valid = false;
            blk = 0;
            it.qb = it.qe = 0;
        } else {
            const int4 e = t.items[bg * t.max_items + ci];
            blk = e.x;
            it.qb = e.y;
            it.qe = e.z;
        }
    }
    it.valid = it.valid && it.qb < it.qe;
    it.ns = it.valid ? (it.qe - it.qb + kQ - 1) / kQ : 0;
    it.j0 = blk * kKeys;
    it.rows = min(kKeys, a.N - it.j0);
    return it;
}

// Persistent: CTA c walks items c, c + grid, c + 2 grid, ... (valid ones only). The load
// ring, the S/T buffers and the dl / dQ hand-offs continue across items (phases counted by
// the CTA's global step index), so the next item's rows and scalars are fetched while the
// current item finishes; an item's K and V wait for the previous item's last MMA, and its
// first dK, dV product for the softmax warps' read of the previous item's sums.
__global__ void __launch_bounds__(kThr, 1) attend_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                 const __grid_constant__ CUtensorMap tmV,
                                                                 const __grid_constant__ CUtensorMap tmQ,
                                                                 const __grid_constant__ CUtensorMap tmDO,
                                                                 const __grid_constant__ CUtensorMap tmQt,
                                                                 const __grid_constant__ CUtensorMap tmDOt,
                                                                 BwdTcArgs t, int gx, int total) {
    const BwdAttendArgs &a = t.a;
    const int Hk = a.H / a.G;
    // the next valid item at or after j, by this CTA's stride (j >= total: none)
    auto next_valid = [&](int j) {
        for (; j < total; j += (int)gridDim.x)
            if (decode_item(t, j, gx).valid) return j;
        return total;
    };
    const int jfirst = next_valid((int)blockIdx.x);
    if (jfirst >= total) return;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = smem_u32(smem);
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + kMiscOff);
    volatile uint32_t *abort_flag = misc + 1;
    int4 *scal = reinterpret_cast<int4 *>(smem + kScOff);
    auto bar = [&](int i) { return sbase + kBarOff + 8u * i; };

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i == kBarFull || i == kBarFull + 1) cnt = 32;
            if (i == kBarStFree || i == kBarStFree + 1 || i == kBarDlFull || i == kBarDqFree || i == kBarDkvFree) cnt = 8;
            if (i >= kBarPair && i < kBarPair + 8) cnt = 64;
            mbar_init(bar(i), cnt);
        }
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(sbase + kMiscOff),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    // bounded wait on work in progress (a.wait_ns of the global timer; zero, a diagnostic:
    // every such wait expires at once); false once the CTA has aborted
    auto wait = [&](uint32_t barrier, uint32_t parity) -> bool {
        if (a.wait_ns > 0) {
            if (mbar_try_wait(barrier, parity)) return true;
            const uint64_t t0 = global_ns();
            for (int it = 0;; ++it) {
                if (mbar_try_wait(barrier, parity)) return true;
                if ((it & 15) == 15) {
                    if (*abort_flag) return false;
                    if ((long long)(global_ns() - t0) > a.wait_ns) break;
                }
            }
        }
        *abort_flag = 1u;
        atomicOr(t.status, 1u);
        return false;
    };
    auto drain_wait = [&](uint32_t barrier, uint32_t parity) {
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(barrier, parity))
            if ((long long)(global_ns() - t0) > kDrainLimitNs) break;
    };
    auto wait_warp = [&](uint32_t barrier, uint32_t parity) -> bool {
        const bool ok = wait(barrier, parity);
        return __all_sync(kFull, ok);
    };
    auto arrive = [&](uint32_t barrier) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(barrier) : "memory");
    };

    if (warp == kLoadWarp || warp == kLoadWarp + 1) {
        // ---------------------------------------------------------------- loads
        const int lw = warp - kLoadWarp;  // 0: Q rows, K and V, and the scalars; 1: dO rows
        const CUtensorMap *tm = lw == 0 ? &tmQ : &tmDO;     // four-row gathers (chunk items)
        const CUtensorMap *tmt = lw == 0 ? &tmQt : &tmDOt;  // 128-row tiles (window items: consecutive queries)
        const uint32_t dst0 = sbase + (lw == 0 ? kQOff : kDOOff) + lane * 512;  // rows 4 lane .. 4 lane + 3
        // the scalars of rows 4 lane + m of a step, as loaded (records, or lse and D_i of window
        // queries): all four loads at once, for the next step before its stage is free
        int4 raw[4];
        auto load_scalars = [&](const BwdItem &it, int s) {
            const int64_t row0 = (int64_t)it.bh * a.N;
            const int q0 = it.qb + s * kQ;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int q = min(q0 + 4 * lane + m, it.qe - 1);
                if (it.chunk) {
                    raw[m] = __ldg(t.recs + row0 * a.topk + q);
                } else {
                    raw[m] = make_int4(q, __float_as_int(__ldg(a.lse + row0 + q)), __float_as_int(__ldg(t.Dv + row0 + q)),
                                       q);
                }
            }
        };
        int g = 0, nit = 0;  // steps and items issued
        int issued[2] = {0, 0};
        bool ok = true;
        BwdItem cur = decode_item(t, jfirst, gx);
        load_scalars(cur, 0);
        for (int j = jfirst; j < total && ok;) {
            const int jn = next_valid(j + (int)gridDim.x);
            const BwdItem nxt = jn < total ? decode_item(t, jn, gx) : cur;
            const int64_t row0 = (int64_t)cur.bh * a.N;
            for (int s = 0; s < cur.ns; ++s, ++g) {
                const int st = g & 1, u = g >> 1;
                if (u > 0 && !(ok = wait_warp(bar(kBarEmpty + st), (u - 1) & 1))) break;
                const int q0 = cur.qb + s * kQ;
                int gy[4];  // rows in the contiguous copies (query 0's row for an unused one, read but ignored)
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int r = 4 * lane + m;
                    int4 sc = raw[m];
                    if (!cur.chunk && !isfinite(__int_as_float(sc.y))) sc.x = -1;
                    if (q0 + r >= cur.qe) sc = make_int4(-1, 0, 0, 0);
                    if (lw == 0) scal[st * kQ + r] = sc;
                    gy[m] = (int)(row0 + (sc.x >= 0 ? sc.w : 0));
                }
                if (cur.chunk) {
                    const uint32_t dst = dst0 + st * 32768;
                    tma_gather4(dst, tm, bar(kBarFull + st), 0, gy[0], gy[1], gy[2], gy[3]);
                    tma_gather4(dst + 16384, tm, bar(kBarFull + st), 64, gy[0], gy[1], gy[2], gy[3]);
                } else if (lane == 0) {  // rows q0 .. q0 + 127: one tile per 64-column half (rows past
                                         // the run are read and ignored; past the array, zero-filled)
                    const uint32_t dst = sbase + (lw == 0 ? kQOff : kDOOff) + st * 32768;
                    tma_load_2d(dst, tmt, bar(kBarFull + st), 0, (int)(row0 + q0));
                    tma_load_2d(dst + 16384, tmt, bar(kBarFull + st), 64, (int)(row0 + q0));
                }
                if (lw == 0) {  // the scalars, and the bytes of both warps' row copies
                    if (lane == 0) mbar_expect_tx(bar(kBarFull + st), 4 * kQ * 128);
                    else arrive(bar(kBarFull + st));
                }
                ++issued[st];
                if (s == 0 && lw == 0) {  // the item's K and V, once the previous item's MMAs are done
                    if (nit > 0 && !(ok = wait_warp(bar(kBarDone), (nit - 1) & 1))) break;
                    if (lane == 0) {
                        mbar_expect_tx(bar(kBarKV), 4 * kKeys * 128);
#pragma unroll
                        for (int x = 0; x < 2; ++x) {
                            tma_load_4d(sbase + kKOff + x * 8192, &tmK, bar(kBarKV), x * 64, cur.j0, cur.hk, cur.b);
                            tma_load_4d(sbase + kVOff + x * 8192, &tmV, bar(kBarKV), x * 64, cur.j0, cur.hk, cur.b);
                        }
                    }
                }
                if (s + 1 < cur.ns) load_scalars(cur, s + 1);
                else if (jn < total) load_scalars(nxt, 0);
            }
            if (!ok) break;
            ++nit;
            j = jn;
            cur = nxt;
        }
        // every copy started lands before the CTA releases its memory
        if (lane == 0) {
            if (lw == 0 && nit > 0) drain_wait(bar(kBarKV), (uint32_t)(nit - 1) & 1u);
            for (int st = 0; st < 2; ++st)
                if (issued[st] > 0) drain_wait(bar(kBarFull + st), (uint32_t)(issued[st] - 1) & 1u);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issue
        const uint32_t idS = idesc_bf16(kQ, kKeys, false);            // K-major A and B
        const uint32_t idKV = idesc_bf16_ab(kDim, kKeys, true, true);  // MN-major A and B
        const uint32_t idQ = idesc_bf16(kQ, kDim, true);              // K-major A, MN-major B
        auto issue_st = [&](int g) {  // S, T of global step g into buffer g % 2
            const int st = g & 1;
            const uint32_t dS = tmem + st * 128, dT = dS + 64;
#pragma unroll
            for (int ks = 0; ks < kDim / 16; ++ks) {
                const uint32_t qo = st * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32;
                const uint32_t ko = (ks >> 2) * 8192 + (ks & 3) * 32;
                mma_ss(dS, smem_desc(sbase + kQOff + qo, 16, 1024), smem_desc(sbase + kKOff + ko, 16, 1024), idS,
                       ks > 0);
                mma_ss(dT, smem_desc(sbase + kDOOff + qo, 16, 1024), smem_desc(sbase + kVOff + ko, 16, 1024), idS,
                       ks > 0);
            }
            mma_commit(bar(kBarStFull + st));
        };
        auto issue_kv = [&](int g, bool first) {  // dK^T (+)= Q^T dl, dV^T (+)= dO^T cv: 16 queries per MMA
            const int st = g & 1;
#pragma unroll
            for (int ks = 0; ks < kQ / 16; ++ks) {
                const uint32_t ro = st * 32768 + ks * 2048;
                const uint32_t acc = (!first || ks > 0) ? 1u : 0u;
                mma_ss(tmem + 256, smem_desc(sbase + kQOff + ro, 16384, 1024),
                       smem_desc(sbase + kDLOff + ks * 2048, 8192, 1024), idKV, acc);
                mma_ss(tmem + 320, smem_desc(sbase + kDOOff + ro, 16384, 1024),
                       smem_desc(sbase + kCVOff + ks * 2048, 8192, 1024), idKV, acc);
            }
            mma_commit(bar(kBarEmpty + st));  // the last reads of the stage's Q and dO rows
        };
        auto issue_dq = [&]() {  // dQ = dl K: 16 keys per MMA
#pragma unroll
            for (int ks = 0; ks < kKeys / 16; ++ks)
                mma_ss(tmem + 384, smem_desc(sbase + kDLOff + ks * 32, 16, 1024),
                       smem_desc(sbase + kKOff + ks * 2048, 8192, 1024), idQ, ks > 0 ? 1u : 0u);
            mma_commit(bar(kBarDqFull));
        };
        // Per item, each product is issued as soon as its inputs are ready, earliest step
        // first within a kind, S/T ahead of the rest: S, T of step n need its rows (full),
        // their TMEM buffer read (the softmax of step n - 2) and the item's K and V; dK, dV
        // of step n need dl, cv of n (and, for the item's first, the softmax warps' read of
        // the previous item's sums); dQ of step n needs dK, dV of n issued and dQ of n - 1
        // read. Every test is a non-blocking look at a phase whose predecessor this warp
        // has already seen.
        bool ok = true;
        int g0 = 0, nit = 0;
        for (int j = jfirst; j < total && ok; j = next_valid(j + (int)gridDim.x)) {
            const BwdItem it = decode_item(t, j, gx);
            if (!(ok = wait_warp(bar(kBarKV), nit & 1))) break;
            int nS = 0, nK = 0, nQ = 0;
            uint64_t idle_since = 0;
            int idle = 0;
            while (ok && nQ < it.ns) {
                int kind = -1;
                if (lane == 0) {
                    const int gS = g0 + nS, gK = g0 + nK, gQ = g0 + nQ;
                    if (nS < it.ns && mbar_test(bar(kBarFull + (gS & 1)), (gS >> 1) & 1) &&
                        (gS < 2 || mbar_test(bar(kBarStFree + (gS & 1)), ((gS >> 1) - 1) & 1)))
                        kind = 0;
                    else if (nK < nS && mbar_test(bar(kBarDlFull), gK & 1) &&
                             (nK > 0 || nit == 0 || mbar_test(bar(kBarDkvFree), (nit - 1) & 1)))
                        kind = 1;
                    else if (nQ < nK && (gQ == 0 || mbar_test(bar(kBarDqFree), (gQ - 1) & 1)))
                        kind = 2;
                }
                kind = __shfl_sync(kFull, kind, 0);
                if (kind >= 0) {
                    tc_fence_after();
                    if (lane == 0) {
                        if (kind == 0) issue_st(g0 + nS);
                        else if (kind == 1) issue_kv(g0 + nK, nK == 0);
                        else issue_dq();
                    }
                    __syncwarp();
                    if (kind == 0) ++nS;
                    else if (kind == 1) ++nK;
                    else ++nQ;
                    idle = 0;
                    continue;
                }
                // nothing ready: bounded like every other wait
                __nanosleep(32);
                if (idle == 0) idle_since = global_ns();
                if ((++idle & 15) == 0 || a.wait_ns <= 0) {
                    bool stop = *abort_flag != 0u;
                    if (!stop && (a.wait_ns <= 0 || (long long)(global_ns() - idle_since) > a.wait_ns)) {
                        *abort_flag = 1u;
                        atomicOr(t.status, 1u);
                        stop = true;
                    }
                    ok = !__any_sync(kFull, stop);
                }
            }
            if (!ok) break;
            if (lane == 0) mma_commit(bar(kBarDone));  // every MMA of the item (dK^T, dV^T final)
            __syncwarp();
            g0 += it.ns;
            ++nit;
        }
        if (lane == 0) {
            // every MMA issued completes before TMEM and shared memory are released
            mma_commit(bar(kBarDrain));
            drain_wait(bar(kBarDrain), 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax rows
        // warp w: rows r = 32 (w % 4) + lane (its TMEM lane quadrant), half g = w / 4 of the
        // keys (columns 32 g .. 32 g + 31 of S and T) and of dQ's columns (64 g .. 64 g + 63);
        // the two halves of a row meet through shared memory (row max, then sum and o_c . dO)
        const int g = warp >> 2, quad = warp & 3;
        const int r = quad * 32 + lane;  // query row of the step = TMEM lane
        const uint32_t lb = (uint32_t)(quad * 32) << 16;
        const float sl2 = a.scale * kLog2e;
        const int K = a.topk;
        float *xm = reinterpret_cast<float *>(smem + kXOff);        // [2][128] half-row maxima
        float2 *xz = reinterpret_cast<float2 *>(smem + kXOff + 1024);  // [2][128] half-row sum, o_c . dO
        // the two warps of a row quadrant (quad and quad + 4) meet on mbarrier kBarPair + 2
        // quad + round (64 arrivals, one phase per chunk step), a bounded wait like every other
        auto pair_sync = [&](int round, int pc) -> bool {
            arrive(bar(kBarPair + 2 * quad + round));
            return wait_warp(bar(kBarPair + 2 * quad + round), pc & 1);
        };
        int64_t prev = -1;  // dQ row (b, h, query) of this row in the previous step, or -1
        // this row's half of the dQ of the last completed step into the global dQ
        auto dq_out = [&](int64_t qrow) {
            float *dst = a.dQ + (qrow < 0 ? 0 : qrow) * kDim + g * 64;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + lb + 384 + g * 64 + c * 32, v);
                tmem_wait_ld();
                if (qrow >= 0) {
                    if (t.vec_ok) {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            atomicAdd(reinterpret_cast<float4 *>(dst + c * 32 + 4 * u),
                                      make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                                  __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3])));
                    } else {
#pragma unroll
                        for (int u = 0; u < 32; ++u) atomicAdd(dst + c * 32 + u, __uint_as_float(v[u]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive(bar(kBarDqFree));
        };
        bool ok = true;
        int gs = 0, pc = 0, nit = 0;  // global step, chunk steps, items
        for (int j = jfirst; j < total && ok; j = next_valid(j + (int)gridDim.x)) {
            const BwdItem it = decode_item(t, j, gx);
            const int j0 = it.j0, rows = it.rows;
            for (int s = 0; s < it.ns; ++s, ++gs) {
                const int st = gs & 1;
                if (!(ok = wait_warp(bar(kBarStFull + st), (gs >> 1) & 1))) break;
                tc_fence_after();
                uint32_t sv[32], tv[32];
                tmem_ld32(tmem + lb + st * 128 + g * 32, sv);
                tmem_ld32(tmem + lb + st * 128 + 64 + g * 32, tv);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive(bar(kBarStFree + st));
                // the step's scalars: their producer's arrival on the stage (complete by now)
                if (!(ok = wait_warp(bar(kBarFull + st), (gs >> 1) & 1))) break;
                const int4 sc = scal[st * kQ + r];
                const int en = sc.x, qi = sc.w;
                const float wl = __int_as_float(sc.y), Dd = __int_as_float(sc.z);
                auto S = [&](int jj) { return __uint_as_float(sv[jj]); };
                auto T = [&](int jj) { return __uint_as_float(tv[jj]); };
                uint32_t dlp[16], cvp[16];  // bf16 pairs of keys 32 g + 2 p, + 1
                if (it.chunk) {
                    // p_j = softmax over the chunk of scale S_j; o_c . dO = sum_j p_j T_j;
                    // dl_j = w p_j (T_j - o_c . dO), cv_j = w p_j; dscore = w (o_c . dO - D_i)
                    float mx[4] = {S(0), S(1), S(2), S(3)};
#pragma unroll
                    for (int jj = 4; jj < 32; ++jj) mx[jj & 3] = fmaxf(mx[jj & 3], S(jj));
                    xm[g * kQ + r] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                    if (!(ok = pair_sync(0, pc))) break;
                    const float ms = fmaxf(xm[r], xm[kQ + r]) * sl2;
                    float e[32], zp[4] = {0.f, 0.f, 0.f, 0.f}, op[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        e[jj] = ex2(fmaf(S(jj), sl2, -ms));
                        zp[jj & 3] += e[jj];
                        op[jj & 3] = fmaf(e[jj], T(jj), op[jj & 3]);
                    }
                    xz[g * kQ + r] = make_float2((zp[0] + zp[1]) + (zp[2] + zp[3]), (op[0] + op[1]) + (op[2] + op[3]));
                    if (!(ok = pair_sync(1, pc))) break;
                    ++pc;
                    const float2 z0 = xz[r], z1 = xz[kQ + r];
                    const float inv = 1.f / (z0.x + z1.x);
                    const float oc = (z0.y + z1.y) * inv;
                    const float wc = en >= 0 ? wl * inv : 0.f;
#pragma unroll
                    for (int p = 0; p < 16; ++p) {
                        const float c0 = wc * e[2 * p], c1 = wc * e[2 * p + 1];
                        cvp[p] = pack_bf16(c0, c1);
                        dlp[p] = pack_bf16(a.scale * c0 * (T(2 * p) - oc), a.scale * c1 * (T(2 * p + 1) - oc));
                    }
                    if (g == 0 && en >= 0) a.dscore[((int64_t)it.bh * a.N + qi) * K + (en & 31)] = wl * (oc - Dd);
                } else {
                    // window key j0 + j of query qi: c_j = exp(scale S_j - lse), dl_j = c_j (T_j - D_i)
                    const float l2 = wl * kLog2e;
#pragma unroll
                    for (int p = 0; p < 16; ++p) {
                        float c[2];
#pragma unroll
                        for (int hv = 0; hv < 2; ++hv) {
                            const int jj = 32 * g + 2 * p + hv, key = j0 + jj;
                            const bool in = en >= 0 && jj < rows && key <= qi && key > qi - a.W;
                            c[hv] = in ? ex2(fmaf(S(2 * p + hv), sl2, -l2)) : 0.f;
                        }
                        cvp[p] = pack_bf16(c[0], c[1]);
                        dlp[p] = pack_bf16(a.scale * c[0] * (T(2 * p) - Dd), a.scale * c[1] * (T(2 * p + 1) - Dd));
                    }
                }
                // dl, cv of the previous step were read by its MMAs once its dQ completed
                if (gs > 0) {
                    if (!(ok = wait_warp(bar(kBarDqFull), (gs - 1) & 1))) break;
                    tc_fence_after();
                }
                uint8_t *dlrow = smem + kDLOff + r * 128, *cvrow = smem + kCVOff + r * 128;
#pragma unroll
                for (int u = 0; u < 4; ++u) {  // 16-byte units 4 g + u of the row (keys 32 g + 8 u ..)
                    const int o = ((4 * g + u) ^ (r & 7)) << 4;
                    *reinterpret_cast<uint4 *>(dlrow + o) = make_uint4(dlp[4 * u], dlp[4 * u + 1], dlp[4 * u + 2], dlp[4 * u + 3]);
                    *reinterpret_cast<uint4 *>(cvrow + o) = make_uint4(cvp[4 * u], cvp[4 * u + 1], cvp[4 * u + 2], cvp[4 * u + 3]);
                }
                asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                __syncwarp();
                if (lane == 0) arrive(bar(kBarDlFull));
                if (gs > 0) dq_out(prev);
                prev = en >= 0 ? (int64_t)it.bh * a.N + qi : -1;
            }
            if (!ok) break;
            // the item's dK^T and dV^T: row r of TMEM is dimension x = r; key j in column j
            // (this warp's half); then the next item's first dK, dV product may overwrite them
            if (!(ok = wait_warp(bar(kBarDone), nit & 1))) break;
            tc_fence_after();
            {
                const int64_t kvrow = ((int64_t)it.b * Hk + it.hk) * a.N + j0;
                float *dk = a.dK + kvrow * kDim + r;
                float *dv = a.dV + kvrow * kDim + r;
                uint32_t vk[32], vv[32];
                tmem_ld32(tmem + lb + 256 + g * 32, vk);
                tmem_ld32(tmem + lb + 320 + g * 32, vv);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive(bar(kBarDkvFree));
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int jj = g * 32 + u;
                    if (jj < rows) {
                        atomicAdd(dk + (int64_t)jj * kDim, __uint_as_float(vk[u]));
                        atomicAdd(dv + (int64_t)jj * kDim, __uint_as_float(vv[u]));
                    }
                }
            }
            ++nit;
        }
        // the last step's dQ (complete: the last item's MMAs were awaited above)
        if (ok && gs > 0) dq_out(prev);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
    }
}

// [rows, 128] contiguous bf16 -> 2-D map with a (64 elements x box_rows) box, 128-byte
// swizzle: one row for four-row gathers, 128 for tiles of consecutive rows.
bool make_row_map(CUtensorMap *m, const void *ptr, int64_t rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kDim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kDim * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

hils_status launch_attend_bwd_tc(const BwdTcArgs &t, const void *Qc, const void *dOb, cudaStream_t s) {
    const BwdAttendArgs &a = t.a;
    const int Hk = a.H / a.G;
    const int64_t nrows = (int64_t)a.B * a.H * a.N;
    const int gx = t.nwin + t.max_items;
    if (gx == 0 || nrows == 0) return HILS_OK;
    CUtensorMap mk, mv, mq, mdo, mqt, mdot;
    if (!make_map(&mk, a.K, a.B, Hk, a.N, kKeys) || !make_map(&mv, a.V, a.B, Hk, a.N, kKeys) ||
        !make_row_map(&mq, Qc, nrows, 1) || !make_row_map(&mdo, dOb, nrows, 1) || !make_row_map(&mqt, Qc, nrows, kQ) ||
        !make_row_map(&mdot, dOb, nrows, kQ))
        return HILS_ERR_CUDA;
    static KernelSetup setup;
    int per_sm = 0;
    const hils_status st = kernel_setup(setup, (const void *)attend_bwd_tc_kernel, kThr, kSmemBytes, &per_sm);
    if (st != HILS_OK) return st;
    if (per_sm < 1) return HILS_ERR_CUDA;
    const int64_t total = (int64_t)gx * a.B * a.H;
    if (total > 0x7fffffffll) return HILS_ERR_UNSUPPORTED;
    const int grid = (int)std::min<int64_t>(total, (int64_t)per_sm * device_sm_count());
    attend_bwd_tc_kernel<<<grid, kThr, kSmemBytes, s>>>(mk, mv, mq, mdo, mqt, mdot, t, gx, (int)total);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace hils
