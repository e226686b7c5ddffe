// Prefill attend on the 5th-generation tensor cores (bf16, d = 128): "Hierarchical
// Sparse Attention Done Right" (picx.dev summary), Methodology 2, Eq. 10, with the
// query-packing kernel of its Efficiency section (adjacent queries share the union of
// their kept chunks, so the per-chunk products are dense tensor-core tiles).
//
// A persistent CTA (one per SM) takes work items of two 128-row query tiles A and B
// that share every key/value tile. A tile packs P query heads that share a key-value
// head and, with grouped-query attention, their kept chunks (the summary page's
// M x G >= 16 packing: P = the largest power of two <= 8 dividing the group size G),
// each with 128 / P consecutive queries; an item covers 2 x 128 / P consecutive
// queries t0.. of those heads (P = 1: 256 queries of one head). Each item walks 64-key
// tiles:
//   1. the window tiles covering [max(0, t0-W+1), last query] (online softmax; a row's
//      reference max is raised, and O rescaled, only when the row's tile max passes it
//      by more than 8 in log2 units);
//   2. the union of the chunks kept by the item's queries, ascending, one chunk per
//      tile; a row that kept chunk c weights that chunk's own softmax by exp(s^_c), a
//      row that did not contributes zero.
// Warp roles (384 threads), all hand-offs through mbarriers:
//   warps 0-3  softmax of tile A (thread = row = TMEM lane), warps 4-7 softmax of B;
//   warp 8     TMA loads (Q of both tiles; K and V of each key tile, 4-slot rings);
//   warps 9/11 tcgen05.mma issue for tile A / tile B: S_X = Q_X K^T (M=128, N=64, K=128)
//              into TMEM, then O_X += P_X V (M=128, N=128, K=64, the A operand P_X read
//              from TMEM); one issuer per tile, so that neither waits on the other's rows;
//   warp 10    builds the next item's union bitmap while the others work.
// S is double-buffered per query tile and P_X(i) is written over S_X(i) (its first 32
// columns): S_X(i+1) is computed while the softmax of tile i runs. A later MMA is not
// ordered after the TMEM operand reads of an earlier one, so the MMA warp issues S_X(i+2)
// into buffer i % 2 only once the completion of PV_X(i), which read P_X(i) there, has
// been signalled on that buffer's barrier; PV_X(i) is issued a whole tile earlier, so the
// wait rarely blocks. A parity wait is exact only while the phase before the awaited one
// has completed; the PV barrier of a buffer is first awaited by the MMA warp (before it
// reuses the buffer), which also makes the softmax's waits for O on it exact.
// TMEM: S_A0 [0,64), S_A1 [64,128), S_B0 [128,192), S_B1 [192,256), O_A [256,384),
// O_B [384,512).
// Every mbarrier wait is bounded in time (the global timer): on expiry the CTA records an
// error in the status word, every role stops issuing work, the CTA drains the copies and
// MMAs it started (each drain wait bounded again), frees its TMEM and exits; outputs of
// unfinished items are not written.
#include "tc_common.cuh"
#include "fast_math.cuh"

namespace hils {
namespace {

using namespace tc;

constexpr int kM = 128;          // query rows per tile
constexpr int kRows = 2 * kM;    // query rows per work item
constexpr int kTile = 64;        // keys per tile (= chunk size)
constexpr int kHead = 128;       // head dimension
constexpr int kSoftmaxWarps = 8;
constexpr int kLoadWarp = 8, kMmaWarp = 9, kMapWarp = 10, kMmaWarpB = 11;
constexpr int kThreads = 384;
constexpr int kStages = 4;       // K/V ring depth
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxBitmapWords = 256;  // union bitmap: up to 8192 chunks

// shared memory map (offsets from the 1024-aligned base)
constexpr int kQOff = 0;                                  // 2 tiles x 2 blocks x [128 rows x 128 B]
constexpr int kKOff = 65536;                              // kStages x 2 blocks x [64 keys x 128 B]
constexpr int kVOff = kKOff + kStages * 16384;            // same
constexpr int kBarOff = kVOff + kStages * 16384;          // mbarriers
constexpr int kMiscOff = kBarOff + 512;                   // tmem base, abort flag, union counts
constexpr int kBitmapOff = kMiscOff + 64;                 // 2 union bitmaps (double-buffered by item)
constexpr int kNselOff = kBitmapOff + 2 * kMaxBitmapWords * 4;  // 2 x [256] kept counts (builder)
constexpr int kSmemBytes = kNselOff + 2 * kRows * 4 + 1024;     // + alignment slack

enum {
    kBarQfull = 0,
    kBarQfree = 1,
    kBarKfull = 2,       // + slot
    kBarKfree = 6,       // + slot
    kBarVfull = 10,      // + slot
    kBarVfree = 14,      // + slot
    kBarSfull = 18,      // + 2 * tile + buffer: S_X written
    kBarPfull = 22,      // + 2 * tile + buffer: P_X written over it
    kBarPVdone = 26,     // + 2 * tile + buffer: the PV that read the buffer (and every MMA
                         //   issued before it) completed
    kBarMapReady = 30,   // + item parity
    kBarMapFree = 32,    // + item parity
    kBarDrain = 34,      // + issuer (A, B)
    kNumBars = 36
};
constexpr uint32_t kMapFreeCount = kSoftmaxWarps * 32 + 3;  // softmax rows + load warp + 2 MMA warps

struct TcArgs {
    AttendArgs a;
    int N, C;
    int nqb;        // query items per (b, packed heads)
    int items;      // B * (H / P) * nqb
    uint32_t *status;  // nonzero after a wait expired
};

// smallest set bit >= from in the bitmap, or -1
__device__ __forceinline__ int next_bit(const uint32_t *bm, int nwords, int from) {
    int w = from >> 5;
    if (w >= nwords || from < 0) return -1;
    uint32_t m = bm[w] & (0xffffffffu << (from & 31));
    while (true) {
        if (m) return (w << 5) + __ffs(m) - 1;
        if (++w >= nwords) return -1;
        m = bm[w];
    }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Loads that the compiler keeps where they are written: a kept-list entry is fetched
// four selections before it is needed, not at its first use.
__device__ __forceinline__ int ldg_early(const int32_t *p) {
    int v;
    asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ float ldg_early(const float *p) {
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// The work item of round r for CTA c: rounds alternate direction so that every CTA gets
// a similar share of the expensive (late-query) items, which come first.
__device__ __forceinline__ int item_of(int r, int c, int G) { return r * G + ((r & 1) ? (G - 1 - c) : c); }

struct Item {
    int b, h, hk, t0;  // batch, first packed query head, their key-value head, first query
    int ws0, nw;  // window: first key, tiles
};

template <int P>
__device__ __forceinline__ Item decode_item(const TcArgs &args, int j) {
    constexpr int kQt = kM / P;
    const AttendArgs &a = args.a;
    const int hp = a.H / P;
    const int units = a.B * hp;
    Item it;
    const int qb = args.nqb - 1 - j / units;  // latest query blocks first
    const int u = j % units;
    it.b = u / hp;
    it.h = (u % hp) * P;
    it.hk = it.h / a.G;
    it.t0 = qb * 2 * kQt;
    it.ws0 = 0;
    it.nw = 0;
    if (a.W > 0) {
        const int lo = max(0, it.t0 - a.W + 1);
        const int hi = min(args.N - 1, it.t0 + 2 * kQt - 1);
        it.ws0 = (lo / kTile) * kTile;
        it.nw = (hi - it.ws0) / kTile + 1;
    }
    return it;
}

template <int P>
__global__ void __launch_bounds__(kThreads, 1) attend_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                         const __grid_constant__ CUtensorMap tmK,
                                                                         const __grid_constant__ CUtensorMap tmV,
                                                                         TcArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const AttendArgs &a = args.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = smem_u32(smem);
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + kMiscOff);
    volatile uint32_t *abort_flag = misc + 1;
    volatile uint32_t *union_count = misc + 2;  // [2], by item parity
    uint32_t *bitmaps = reinterpret_cast<uint32_t *>(smem + kBitmapOff);
    const int nwords = (args.C + 31) >> 5;
    auto bar = [&](int i) { return sbase + kBarOff + 8u * i; };
    const int G = gridDim.x, cta = blockIdx.x;
    constexpr int kQt = kM / P;  // queries per packed head and tile

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i >= kBarPfull && i < kBarPfull + 4) cnt = 4;  // one elected lane per softmax warp
            if (i == kBarQfree || (i >= kBarKfree && i < kBarKfree + kStages) ||
                (i >= kBarVfree && i < kBarVfree + kStages))
                cnt = 2;  // both MMA issuers release shared operands
            if (i == kBarMapReady || i == kBarMapReady + 1) cnt = 32;
            if (i == kBarMapFree || i == kBarMapFree + 1) cnt = kMapFreeCount;
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
    // every such wait expires at once); false once the CTA has aborted (the first expiry
    // sets the flag)
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
        atomicOr(args.status, 1u);
        return false;
    };
    // bounded wait for a phase of this CTA's own copies or MMAs while it stops
    auto drain_wait = [&](uint32_t barrier, uint32_t parity) {
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(barrier, parity))
            if ((long long)(global_ns() - t0) > kDrainLimitNs) break;
    };
    // warp-uniform form: every lane waits, the warp goes on only if all succeeded
    auto wait_warp = [&](uint32_t barrier, uint32_t parity) -> bool {
        const bool ok = wait(barrier, parity);
        return __all_sync(kFull, ok);
    };
    auto arrive = [&](uint32_t barrier) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(barrier) : "memory");
    };

    const float kLog2e = 1.4426950408889634f;
    const float scale2 = a.scale * kLog2e;

    if (warp == kMapWarp) {
        // ---------------------------------------------------------------- union builder
        for (int r = 0, n = 0;; ++r, ++n) {
            const int j = item_of(r, cta, G);
            if (j >= args.items) break;
            const Item it = decode_item<P>(args, j);
            const int par = n & 1;
            if (n >= 2 && !wait_warp(bar(kBarMapFree + par), ((n - 2) >> 1) & 1)) break;
            uint32_t *bm = bitmaps + par * kMaxBitmapWords;
            int *nsm = reinterpret_cast<int *>(smem + kNselOff) + par * kRows;
            for (int i = lane; i < nwords; i += 32) bm[i] = 0u;
            // the item's queries are consecutive: their kept lists form one contiguous block,
            // read with many loads in flight
            const int nrows = min(2 * kQt, args.N - it.t0);
            const int64_t q0 = ((int64_t)it.b * (a.H / a.G) + it.hk) * a.Lq + it.t0;  // the group's kept lists
#pragma unroll
            for (int rr = lane; rr < kRows; rr += 32)
                nsm[rr] = (a.topk > 0 && rr < nrows) ? min(max(__ldg(&a.nsel[q0 + rr]), 0), a.topk) : 0;
            __syncwarp();
            const int tot = a.topk > 0 ? nrows * a.topk : 0;
            const int32_t *ib = a.idx + q0 * a.topk;
            for (int e0 = 0; e0 < tot; e0 += 32 * 16) {
                int cv[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int e = e0 + u * 32 + lane;
                    cv[u] = e < tot ? __ldg(&ib[e]) : -1;
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int e = e0 + u * 32 + lane;
                    if (cv[u] >= 0 && cv[u] < args.C) {
                        const int row = e / a.topk;
                        if (e - row * a.topk < nsm[row]) atomicOr(&bm[cv[u] >> 5], 1u << (cv[u] & 31));
                    }
                }
            }
            __syncwarp();
            int cnt = 0;
            for (int i = lane; i < nwords; i += 32) cnt += __popc(bm[i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(kFull, cnt, o);
            if (lane == 0) union_count[par] = (uint32_t)cnt;
            __syncwarp();
            arrive(bar(kBarMapReady + par));
        }
    } else if (warp == kLoadWarp) {
        // ---------------------------------------------------------------- TMA loads
        int g = 0, qn = 0;
        int issuedQ = 0, issuedK = 0, issuedV = 0;  // copies started, in ring order
        for (int r = 0, n = 0;; ++r, ++n) {
            const int j = item_of(r, cta, G);
            if (j >= args.items) break;
            const Item it = decode_item<P>(args, j);
            const int par = n & 1;
            if (!wait_warp(bar(kBarMapReady + par), (n >> 1) & 1)) break;
            const int nt = it.nw + (int)union_count[par];
            const uint32_t *bm = bitmaps + par * kMaxBitmapWords;
            bool ok = true;
            if (nt > 0) {
                if (qn > 0) ok = wait_warp(bar(kBarQfree), (qn - 1) & 1);
                if (!ok) break;
                if (lane == 0) {
                    ++issuedQ;
                    mbar_expect_tx(bar(kBarQfull), 4 * kM * 128);
                    // rows [hh * qt, (hh + 1) * qt) of tile x: head h + hh, queries t0 + x * qt ..
#pragma unroll
                    for (int x = 0; x < 2; ++x)
#pragma unroll
                        for (int hh = 0; hh < P; ++hh)
#pragma unroll
                            for (int kb = 0; kb < 2; ++kb)
                                tma_load_4d(sbase + kQOff + x * 32768 + kb * 16384 + hh * kQt * 128, &tmQ,
                                            bar(kBarQfull), kb * 64, it.t0 + x * kQt, it.h + hh, it.b);
                }
                ++qn;
                int cur = -1;  // union walk
                for (int i = 0; i < nt && ok; ++i, ++g) {
                    int k0;
                    if (i < it.nw) {
                        k0 = it.ws0 + kTile * i;
                    } else {
                        cur = next_bit(bm, nwords, cur + 1);
                        k0 = cur * kTile;
                    }
                    const int s = g % kStages, u = g / kStages;
                    if (u > 0 && !(ok = wait_warp(bar(kBarKfree + s), (u - 1) & 1))) break;
                    if (lane == 0) {
                        ++issuedK;
                        mbar_expect_tx(bar(kBarKfull + s), 2 * kTile * 128);
                        const uint32_t dst = sbase + kKOff + s * 16384;
                        tma_load_4d(dst, &tmK, bar(kBarKfull + s), 0, k0, it.hk, it.b);
                        tma_load_4d(dst + 8192, &tmK, bar(kBarKfull + s), 64, k0, it.hk, it.b);
                    }
                    if (u > 0 && !(ok = wait_warp(bar(kBarVfree + s), (u - 1) & 1))) break;
                    if (lane == 0) {
                        ++issuedV;
                        mbar_expect_tx(bar(kBarVfull + s), 2 * kTile * 128);
                        const uint32_t dst = sbase + kVOff + s * 16384;
                        tma_load_4d(dst, &tmV, bar(kBarVfull + s), 0, k0, it.hk, it.b);
                        tma_load_4d(dst + 8192, &tmV, bar(kBarVfull + s), 64, k0, it.hk, it.b);
                    }
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) arrive(bar(kBarMapFree + par));
        }
        // every copy this warp started lands before the CTA releases its memory (after a
        // normal finish every one was awaited by the MMA warps, so this returns at once)
        if (lane == 0) {
            auto drain = [&](uint32_t b, int issued) {
                if (issued == 0) return;
                drain_wait(b, (uint32_t)(issued - 1) & 1u);
            };
            drain(bar(kBarQfull), issuedQ);
            for (int s = 0; s < kStages; ++s) {  // uses of slot s among the first n ring entries
                drain(bar(kBarKfull + s), issuedK > s ? (issuedK - s + kStages - 1) / kStages : 0);
                drain(bar(kBarVfull + s), issuedV > s ? (issuedV - s + kStages - 1) / kStages : 0);
            }
        }
    } else if (warp == kMmaWarp || warp == kMmaWarpB) {
        // ---------------------------------------------------------------- MMA issue (tile xm)
        const int xm = warp == kMmaWarp ? 0 : 1;
        const uint32_t idS = idesc_bf16(kM, kTile, false);
        const uint32_t idPV = idesc_bf16(kM, kHead, true);
        auto issue_s = [&](int x, int gt) {  // S_x(gt) = Q_x K^T into buffer gt % 2
            const int s = gt % kStages;
            const uint32_t d = tmem + x * 128 + (gt & 1) * 64;
#pragma unroll
            for (int ks = 0; ks < kHead / 16; ++ks) {
                const uint32_t qa = sbase + kQOff + x * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32;
                const uint32_t ka = sbase + kKOff + s * 16384 + (ks >> 2) * 8192 + (ks & 3) * 32;
                mma_ss(d, smem_desc(qa, 16, 1024), smem_desc(ka, 16, 1024), idS, ks > 0);
            }
            mma_commit(bar(kBarSfull + 2 * x + (gt & 1)));
        };
        auto issue_pv = [&](int x, int gt, bool acc) {  // O_x (+)= P_x(gt) V
            const int s = gt % kStages;
#pragma unroll
            for (int ks = 0; ks < kTile / 16; ++ks) {
                const uint32_t va = sbase + kVOff + s * 16384 + ks * 2048;
                mma_ts(tmem + 256 + x * 128, tmem + x * 128 + (gt & 1) * 64 + ks * 8, smem_desc(va, 8192, 1024),
                       idPV, (acc || ks > 0) ? 1u : 0u);
            }
            mma_commit(bar(kBarPVdone + 2 * x + (gt & 1)));
        };
        // S_x(gt) goes into the buffer that PV_x(gt - 2) read: that PV has completed
        auto s_free = [&](int x, int gt) {
            return gt < 2 || wait_warp(bar(kBarPVdone + 2 * x + (gt & 1)), ((gt >> 1) - 1) & 1);
        };
        int g = 0, qn = 0;
        bool ok = true;
        for (int r = 0, n = 0; ok; ++r, ++n) {
            const int j = item_of(r, cta, G);
            if (j >= args.items) break;
            const Item it = decode_item<P>(args, j);
            const int par = n & 1;
            if (!(ok = wait_warp(bar(kBarMapReady + par), (n >> 1) & 1))) break;
            const int nt = it.nw + (int)union_count[par];
            __syncwarp();
            if (lane == 0) arrive(bar(kBarMapFree + par));
            if (nt == 0) continue;
            if (!(ok = wait_warp(bar(kBarQfull), qn & 1))) break;
            ++qn;
            tc_fence_after();
            auto s_one = [&](int gt, bool last) -> bool {  // S_xm(gt)
                if (!wait_warp(bar(kBarKfull + gt % kStages), (gt / kStages) & 1)) return false;
                if (!s_free(xm, gt)) return false;
                tc_fence_after();
                if (lane == 0) {
                    issue_s(xm, gt);
                    mma_commit(bar(kBarKfree + gt % kStages));
                    if (last) mma_commit(bar(kBarQfree));
                }
                __syncwarp();
                return true;
            };
            // S of the item's first two tiles, then per tile: PV of this one, S of the one two ahead
            if (!(ok = s_one(g, nt == 1))) break;
            if (nt > 1 && !(ok = s_one(g + 1, nt == 2))) break;
            for (int i = 0; i < nt; ++i, ++g) {
                if (!(ok = wait_warp(bar(kBarPfull + 2 * xm + (g & 1)), (g >> 1) & 1))) break;
                if (!(ok = wait_warp(bar(kBarVfull + g % kStages), (g / kStages) & 1))) break;
                tc_fence_after();
                if (lane == 0) {
                    issue_pv(xm, g, i > 0);
                    mma_commit(bar(kBarVfree + g % kStages));
                }
                __syncwarp();
                if (i + 2 < nt && !(ok = s_one(g + 2, i + 3 == nt))) break;
            }
        }
        // every MMA this warp issued completes before TMEM and shared memory are released
        if (lane == 0) {
            mma_commit(bar(kBarDrain + xm));
            drain_wait(bar(kBarDrain + xm), 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax rows
        const int x = warp >> 2;            // query tile A (0) or B (1)
        const int quad = warp & 3;          // TMEM lane quadrant
        const int rloc = quad * 32 + lane;  // row within the tile = TMEM lane
        const int hrow = rloc / kQt;        // its packed head
        const int trow = rloc % kQt;        // and query within the tile
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const uint32_t o_col = tmem + lane_base + 256 + x * 128;
        int g = 0;  // key tiles processed, over all items
        for (int r = 0, n = 0;; ++r, ++n) {
            const int j = item_of(r, cta, G);
            if (j >= args.items) break;
            const Item it = decode_item<P>(args, j);
            const int par = n & 1;
            const int t = it.t0 + x * kQt + trow;
            const bool row_ok = t < args.N;
            const int64_t qrow = ((int64_t)it.b * a.H + it.h + hrow) * a.Lq + t;
            const int64_t qgrp = ((int64_t)it.b * (a.H / a.G) + it.hk) * a.Lq + t;  // the group's kept list
            const int nsel = (row_ok && a.topk > 0) ? min(max(__ldg(&a.nsel[qgrp]), 0), a.topk) : 0;
            const int32_t *ip = a.idx + qgrp * a.topk;
            const float *sp = a.score + qrow * a.topk;
            float ref = -INFINITY;  // log2-domain reference: the largest kept chunk score
#pragma unroll 8
            for (int k = 0; k < nsel; ++k) {
                const int c = __ldg(&ip[k]);
                const float sc = __ldg(&sp[k]);
                ref = fmaxf(ref, (c >= 0 && c < args.C) ? sc * kLog2e : -INFINITY);
            }
            // the row's kept list, four entries ahead (ascending chunk indices)
            int qc[4];
            float qs[4];
            int kn = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                qc[e] = kn < nsel ? __ldg(&ip[kn]) : INT_MAX;
                qs[e] = kn < nsel ? __ldg(&sp[kn]) * kLog2e : 0.f;
                ++kn;
            }
            if (!wait_warp(bar(kBarMapReady + par), (n >> 1) & 1)) break;
            const int nt = it.nw + (int)union_count[par];
            const uint32_t *bm = bitmaps + par * kMaxBitmapWords;
            float m_used = ref;
            float l = 0.f;
            int cur = -1;
            bool ok = true;
            for (int i = 0; i < nt; ++i, ++g) {
                const int bsel = g & 1;
                if (!(ok = wait_warp(bar(kBarSfull + 2 * x + bsel), (g >> 1) & 1))) break;
                tc_fence_after();
                const uint32_t s_col = tmem + lane_base + x * 128 + bsel * 64;
                uint32_t sr[64];  // S of this row, then (packed in place into sr[0..31]) its P
                bool any = true;
                if (i < it.nw) {
                    // ---- window tile: keys [ks, ks + 64); valid offsets [jlo, jhi] of this row
                    const int ks = it.ws0 + kTile * i;
                    int jlo = max(0, t - a.W + 1 - ks);
                    int jhi = min(kTile - 1, t - ks);
                    if (!row_ok) {
                        jlo = kTile;
                        jhi = -1;
                    }
                    const bool full = __all_sync(kFull, jlo == 0 && jhi == kTile - 1);
                    any = __any_sync(kFull, jlo <= jhi);
                    if (any) {
                        tmem_ld32(s_col, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                        tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                        tmem_wait_ld();
                    }
                    if (any) {
                        if (!full) {
#pragma unroll
                            for (int q = 0; q < 64; ++q) {
                                const bool v = q >= jlo && q <= jhi;
                                sr[q] = v ? sr[q] : __float_as_uint(-INFINITY);
                            }
                        }
                        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
                        for (int q = 0; q < 64; q += 8) {
                            m0 = max3(m0, __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]));
                            m1 = max3(m1, __uint_as_float(sr[q + 2]), __uint_as_float(sr[q + 3]));
                            m2 = max3(m2, __uint_as_float(sr[q + 4]), __uint_as_float(sr[q + 5]));
                            m3 = max3(m3, __uint_as_float(sr[q + 6]), __uint_as_float(sr[q + 7]));
                        }
                        const float mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * scale2;
                        // raise the row's reference when its tile max passes it by more than 8
                        const bool raise = mt != -INFINITY && (m_used == -INFINITY || mt > m_used + 8.f);
                        const float f = raise ? ex2(m_used - mt) : 1.f;  // 0 when m_used is -inf
                        if (__any_sync(kFull, raise && l > 0.f)) {
                            // O holds earlier tiles of this item: PV_x of the previous tile completes first
                            if (!(ok = wait_warp(bar(kBarPVdone + 2 * x + ((g - 1) & 1)), ((g - 1) >> 1) & 1))) break;
                            tc_fence_after();
                            // in 8-column pieces: S stays in registers meanwhile
#pragma unroll 1
                            for (int part = 0; part < 16; ++part) {
                                uint32_t o[8];
                                tmem_ld8(o_col + part * 8, o);
                                tmem_wait_ld();
#pragma unroll
                                for (int q = 0; q < 8; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * f);
                                tmem_st8(o_col + part * 8, o);
                            }
                        }
                        if (raise) {
                            l *= f;
                            m_used = mt;
                        }
                        const float nb = m_used == -INFINITY ? 0.f : -m_used;
                        float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
                        for (int q = 0; q < 64; q += 4) {
                            const float e0 = ex2(fmaf(__uint_as_float(sr[q]), scale2, nb));
                            const float e1 = ex2(fmaf(__uint_as_float(sr[q + 1]), scale2, nb));
                            const float e2 = ex2(fmaf(__uint_as_float(sr[q + 2]), scale2, nb));
                            const float e3 = ex2(fmaf(__uint_as_float(sr[q + 3]), scale2, nb));
                            z0 += e0;
                            z1 += e1;
                            z2 += e2;
                            z3 += e3;
                            sr[q >> 1] = pack_bf16(e0, e1);  // sr[q/2 + 1] <= sr[q + 1]: already read
                            sr[(q >> 1) + 1] = pack_bf16(e2, e3);
                        }
                        l += (z0 + z1) + (z2 + z3);
                    }
                } else {
                    // ---- chunk tile: the next chunk of the union
                    cur = next_bit(bm, nwords, cur + 1);
                    const int c = cur;
                    const bool sel = row_ok && c >= 0 && qc[0] == c;
                    float wgt = 0.f;
                    if (sel) {
                        wgt = exp2_fma(qs[0] - m_used);  // no MUFU: it would queue behind the exp bursts
                        l += wgt;
                        qc[0] = qc[1];
                        qs[0] = qs[1];
                        qc[1] = qc[2];
                        qs[1] = qs[2];
                        qc[2] = qc[3];
                        qs[2] = qs[3];
                        qc[3] = INT_MAX;
                        qs[3] = 0.f;
                        if (kn < nsel) {
                            qc[3] = ldg_early(ip + kn);
                            qs[3] = ldg_early(sp + kn) * kLog2e;
                        }
                        ++kn;
                    }
                    any = __any_sync(kFull, sel);
                    if (any) {
                        tmem_ld32(s_col, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                        tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                        tmem_wait_ld();
                    }
                    if (any) {
                        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
                        for (int q = 0; q < 64; q += 8) {
                            m0 = max3(m0, __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]));
                            m1 = max3(m1, __uint_as_float(sr[q + 2]), __uint_as_float(sr[q + 3]));
                            m2 = max3(m2, __uint_as_float(sr[q + 4]), __uint_as_float(sr[q + 5]));
                            m3 = max3(m3, __uint_as_float(sr[q + 6]), __uint_as_float(sr[q + 7]));
                        }
                        const float nb = -fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * scale2;
                        float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
                        for (int q = 0; q < 64; q += 4) {
                            const float e0 = ex2(fmaf(__uint_as_float(sr[q]), scale2, nb));
                            const float e1 = ex2(fmaf(__uint_as_float(sr[q + 1]), scale2, nb));
                            const float e2 = ex2(fmaf(__uint_as_float(sr[q + 2]), scale2, nb));
                            const float e3 = ex2(fmaf(__uint_as_float(sr[q + 3]), scale2, nb));
                            z0 += e0;
                            z1 += e1;
                            z2 += e2;
                            z3 += e3;
                            sr[q] = __float_as_uint(e0);
                            sr[q + 1] = __float_as_uint(e1);
                            sr[q + 2] = __float_as_uint(e2);
                            sr[q + 3] = __float_as_uint(e3);
                        }
                        // z >= 1 (the max term is 1): its reciprocal on the FMA pipe
                        const float fw = sel ? wgt * recip_newton((z0 + z1) + (z2 + z3)) : 0.f;
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            sr[q] = pack_bf16(__uint_as_float(sr[2 * q]) * fw, __uint_as_float(sr[2 * q + 1]) * fw);
                    }
                }
                if (!ok) break;
                if (!any) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) sr[q] = 0u;
                }
                tmem_st32(s_col, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive(bar(kBarPfull + 2 * x + bsel));
            }
            // ---- epilogue: O / l and lse
            if (ok && nt > 0) ok = wait_warp(bar(kBarPVdone + 2 * x + ((g - 1) & 1)), ((g - 1) >> 1) & 1);
            if (!ok) break;
            tc_fence_after();
            bf16 *orow = static_cast<bf16 *>(a.O.ptr) + it.b * a.O.sb + (it.h + hrow) * a.O.sh + (int64_t)t * a.O.st;
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                uint32_t o[32];
                if (nt > 0) {  // warp-uniform: every lane loads, rows past N are not stored
                    tmem_ld32(o_col + part * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) o[q] = 0u;
                }
                if (row_ok) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + part * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
                        dst[q] = v;
                    }
                }
            }
            if (row_ok && a.lse) a.lse[qrow] = l > 0.f ? (m_used + log2f(l)) / kLog2e : -INFINITY;
            tc_fence_before();
            arrive(bar(kBarMapFree + par));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace

bool attend_prefill_tc_supported(hils_dtype dt, int d, int N) {
    const int C = N / kChunk;
    return dt == HILS_BF16 && d == kHead && (C + 31) / 32 <= kMaxBitmapWords && N > 0;
}

hils_status launch_attend_prefill_tc(const AttendArgs &a, int N, uint32_t *status, cudaStream_t s) {
    CUtensorMap mq, mk, mv;
    const int Hk = a.H / a.G;
    int P = 1;  // heads packed per tile: the largest power of two <= 8 dividing G
    while (P < 8 && a.G % (2 * P) == 0) P *= 2;
    const int qt = kM / P;
    if (!make_map(&mq, a.Q, a.B, a.H, N, qt) || !make_map(&mk, a.K, a.B, Hk, N, kTile) ||
        !make_map(&mv, a.V, a.B, Hk, N, kTile))
        return HILS_ERR_CUDA;
    static KernelSetup setups[4];
    const void *fns[4] = {(const void *)attend_prefill_tc_kernel<1>, (const void *)attend_prefill_tc_kernel<2>,
                          (const void *)attend_prefill_tc_kernel<4>, (const void *)attend_prefill_tc_kernel<8>};
    const int pi = P == 1 ? 0 : P == 2 ? 1 : P == 4 ? 2 : 3;
    int per_sm = 0;
    const hils_status st = kernel_setup(setups[pi], fns[pi], kThreads, kSmemBytes, &per_sm);
    if (st != HILS_OK) return st;
    if (per_sm < 1) return HILS_ERR_CUDA;
    TcArgs ta;
    ta.a = a;
    ta.N = N;
    ta.C = N / kChunk;
    ta.nqb = (N + 2 * qt - 1) / (2 * qt);
    ta.items = a.B * (a.H / P) * ta.nqb;
    ta.status = status;
    const int grid = min(ta.items, per_sm * device_sm_count());
    switch (P) {
    case 1: attend_prefill_tc_kernel<1><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, ta); break;
    case 2: attend_prefill_tc_kernel<2><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, ta); break;
    case 4: attend_prefill_tc_kernel<4><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, ta); break;
    default: attend_prefill_tc_kernel<8><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, ta); break;
    }
    return record_cuda_error(cudaGetLastError());
}

}  // namespace hils
