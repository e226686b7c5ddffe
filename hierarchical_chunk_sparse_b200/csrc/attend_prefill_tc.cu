// Prefill attend on the 5th-generation tensor cores (bf16, d = 128): "Hierarchical
// Sparse Attention Done Right" (picx.dev summary), Methodology 2, Eq. 10, with the
// query-packing kernel of its Efficiency section (adjacent queries share the union of
// their kept chunks, so the per-chunk products are dense tensor-core tiles).
//
// A persistent CTA (one per SM) takes work items of 256 consecutive queries of one
// (b, h): two 128-row query tiles A and B that share every key/value tile. Each item
// walks 128-key tiles made of two 64-key halves:
//   1. window tiles covering [max(0, t0-W+1), t0+255] (online softmax; a row's
//      reference max is raised, and O rescaled, only when the row's tile max passes it
//      by more than 8 in log2 units);
//   2. the union of the chunks kept by the item's 256 queries, ascending, two chunks per
//      tile; a row that kept chunk c weights that chunk's own softmax by exp(s^_c), a
//      row that did not contributes zero.
// Warp roles (352 threads), all hand-offs through mbarriers:
//   warps 0-3  softmax of tile A (thread = row = TMEM lane), warps 4-7 softmax of B;
//   warp 8     TMA loads (Q of both tiles, K and V of each 128-key tile, 2-slot ring);
//   warp 9     tcgen05.mma issue: S_X = Q_X K^T (M=128, N=128, K=128) into TMEM, then
//              O_X += P_X V (A operand P_X read from TMEM over the columns of S_X);
//   warp 10    builds the next item's union bitmap while the others work.
// The MMA warp alternates the two tiles (S_A(i), PV_B(i-1), S_B(i), PV_A(i), ...), so
// the softmax of one tile runs while the tensor pipe works on the other. The tensor
// pipe executes one thread's tcgen05.mma in issue order, which is what lets S_X(i+1)
// reuse the TMEM columns of P_X(i) once PV_X(i) has been issued. TMEM: S_A [0,128),
// S_B [128,256), O_A [256,384), O_B [384,512).
// Every mbarrier wait is bounded: on expiry the CTA records an error in the status word,
// every role stops issuing work, the CTA drains the copies and MMAs it started, frees
// its TMEM and exits; outputs of unfinished items are not written.
#include "tc_common.cuh"

namespace hils {
namespace {

using namespace tc;

constexpr int kM = 128;          // query rows per tile
constexpr int kRows = 2 * kM;    // query rows per work item
constexpr int kHalf = 64;        // keys per half tile (= chunk size)
constexpr int kHead = 128;       // head dimension
constexpr int kSoftmaxThreads = 256;
constexpr int kLoadWarp = 8, kMmaWarp = 9, kMapWarp = 10;
constexpr int kThreads = 352;
constexpr int kStages = 2;       // K/V ring depth
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxBitmapWords = 256;  // union bitmap: up to 8192 chunks
constexpr long long kWaitLimit = 1ll << 26;

// shared memory map (offsets from the 1024-aligned base)
constexpr int kQOff = 0;                                  // 2 tiles x 2 blocks x [128 rows x 128 B]
constexpr int kKOff = 65536;                              // kStages x 2 blocks x [128 keys x 128 B]
constexpr int kVOff = kKOff + kStages * 32768;            // same
constexpr int kBarOff = kVOff + kStages * 32768;          // mbarriers
constexpr int kMiscOff = kBarOff + 256;                   // tmem base, abort flag, union counts
constexpr int kBitmapOff = kMiscOff + 64;                 // 2 union bitmaps (double-buffered by item)
constexpr int kSmemBytes = kBitmapOff + 2 * kMaxBitmapWords * 4 + 1024;  // + alignment slack

enum {
    kBarQfull = 0,
    kBarQfree = 1,
    kBarKfull = 2,   // + slot
    kBarKfree = 4,   // + slot
    kBarVfull = 6,   // + slot
    kBarVfree = 8,   // + slot
    kBarSfull = 10,  // + tile (A, B)
    kBarPfull = 12,  // + tile
    kBarOdone = 14,  // + tile
    kBarMapReady = 16,  // + item parity
    kBarMapFree = 18,   // + item parity
    kBarDrain = 20,
    kNumBars = 21
};
constexpr uint32_t kMapFreeCount = kSoftmaxThreads + 2;  // softmax rows + load warp + MMA warp

struct TcArgs {
    AttendArgs a;
    int N, C;
    int nqb;        // query items per (b, h)
    int items;      // B * H * nqb
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

// The work item of round r for CTA c: rounds alternate direction so that every CTA gets
// a similar share of the expensive (late-query) items, which come first.
__device__ __forceinline__ int item_of(int r, int c, int G) { return r * G + ((r & 1) ? (G - 1 - c) : c); }

struct Item {
    int b, h, t0;
    int ws0, nhw, nwt;  // window: first key, halves, tiles
};

__device__ __forceinline__ Item decode_item(const TcArgs &args, int j) {
    const AttendArgs &a = args.a;
    const int BH = a.B * a.H;
    Item it;
    const int qb = args.nqb - 1 - j / BH;  // latest query blocks first
    const int bh = j % BH;
    it.b = bh / a.H;
    it.h = bh % a.H;
    it.t0 = qb * kRows;
    it.ws0 = 0;
    it.nhw = 0;
    if (a.W > 0) {
        const int lo = max(0, it.t0 - a.W + 1);
        const int hi = min(args.N - 1, it.t0 + kRows - 1);
        it.ws0 = (lo / kHalf) * kHalf;
        it.nhw = (hi - it.ws0) / kHalf + 1;
    }
    it.nwt = (it.nhw + 1) >> 1;
    return it;
}

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

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i == kBarPfull || i == kBarPfull + 1) cnt = kM;
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

    // bounded wait; false once the CTA has aborted (the first expiry sets the flag)
    auto wait = [&](uint32_t barrier, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        for (long long it = 0; it < kWaitLimit; ++it) {
            if (mbar_try_wait(barrier, parity)) return true;
            if ((it & 255) == 255 && *abort_flag) return false;
        }
        *abort_flag = 1u;
        atomicOr(args.status, 1u);
        return false;
    };
    // warp-uniform form: every lane waits, the warp goes on only if all succeeded
    auto wait_warp = [&](uint32_t barrier, uint32_t parity) -> bool {
        const bool ok = wait(barrier, parity);
        return __all_sync(kFull, ok);
    };

    const float kLog2e = 1.4426950408889634f;
    const float scale2 = a.scale * kLog2e;

    if (warp == kMapWarp) {
        // ---------------------------------------------------------------- union builder
        for (int r = 0, n = 0;; ++r, ++n) {
            const int j = item_of(r, cta, G);
            if (j >= args.items) break;
            const Item it = decode_item(args, j);
            const int par = n & 1;
            if (n >= 2 && !wait_warp(bar(kBarMapFree + par), ((n - 2) >> 1) & 1)) break;
            uint32_t *bm = bitmaps + par * kMaxBitmapWords;
            for (int i = lane; i < nwords; i += 32) bm[i] = 0u;
            __syncwarp();
            if (a.topk > 0) {
                for (int rr = lane; rr < kRows; rr += 32) {
                    const int t = it.t0 + rr;
                    if (t >= args.N) break;
                    const int64_t qrow = ((int64_t)it.b * a.H + it.h) * a.Lq + t;
                    const int ns = min(max(__ldg(&a.nsel[qrow]), 0), a.topk);
                    const int32_t *ip = a.idx + qrow * a.topk;
                    for (int k = 0; k < ns; ++k) {
                        const int c = __ldg(&ip[k]);
                        if (c >= 0 && c < args.C) atomicOr(&bm[c >> 5], 1u << (c & 31));
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
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar(kBarMapReady + par)) : "memory");
        }
    } else if (warp == kLoadWarp) {
        // ---------------------------------------------------------------- TMA loads
        int g = 0, qn = 0;
        int issuedQ = 0, issuedK = 0, issuedV = 0;  // copies started, in ring order
        for (int r = 0, n = 0;; ++r, ++n) {
            const int j = item_of(r, cta, G);
            if (j >= args.items) break;
            const Item it = decode_item(args, j);
            const int par = n & 1;
            if (!wait_warp(bar(kBarMapReady + par), (n >> 1) & 1)) break;
            const int nu = (int)union_count[par];
            const int nt = it.nwt + ((nu + 1) >> 1);
            const uint32_t *bm = bitmaps + par * kMaxBitmapWords;
            bool ok = true;
            if (nt > 0) {
                if (qn > 0) ok = wait_warp(bar(kBarQfree), (qn - 1) & 1);
                if (!ok) break;
                if (lane == 0) {
                    ++issuedQ;
                    mbar_expect_tx(bar(kBarQfull), 4 * kM * 128);
#pragma unroll
                    for (int x = 0; x < 2; ++x)
#pragma unroll
                        for (int kb = 0; kb < 2; ++kb)
                            tma_load_4d(sbase + kQOff + x * 32768 + kb * 16384, &tmQ, bar(kBarQfull), kb * 64,
                                        it.t0 + x * kM, it.h, it.b);
                }
                ++qn;
                int cur = -1;  // union walk
                for (int i = 0; i < nt && ok; ++i, ++g) {
                    int k0, k1;
                    if (i < it.nwt) {
                        k0 = it.ws0 + kHalf * (2 * i);
                        k1 = it.ws0 + kHalf * min(2 * i + 1, it.nhw - 1);
                    } else {
                        const int c0 = next_bit(bm, nwords, cur + 1);
                        const int c1 = next_bit(bm, nwords, c0 + 1);
                        cur = c1 >= 0 ? c1 : c0;
                        k0 = c0 * kHalf;
                        k1 = (c1 >= 0 ? c1 : c0) * kHalf;
                    }
                    const int s = g % kStages, u = g / kStages;
                    if (u > 0 && !(ok = wait_warp(bar(kBarKfree + s), (u - 1) & 1))) break;
                    if (lane == 0) {
                        ++issuedK;
                        mbar_expect_tx(bar(kBarKfull + s), 4 * kHalf * 128);
                        const uint32_t dst = sbase + kKOff + s * 32768;
#pragma unroll
                        for (int kb = 0; kb < 2; ++kb) {
                            tma_load_4d(dst + kb * 16384, &tmK, bar(kBarKfull + s), kb * 64, k0, it.h, it.b);
                            tma_load_4d(dst + kb * 16384 + 8192, &tmK, bar(kBarKfull + s), kb * 64, k1, it.h, it.b);
                        }
                    }
                    if (u > 0 && !(ok = wait_warp(bar(kBarVfree + s), (u - 1) & 1))) break;
                    if (lane == 0) {
                        ++issuedV;
                        mbar_expect_tx(bar(kBarVfull + s), 4 * kHalf * 128);
                        const uint32_t dst = sbase + kVOff + s * 32768;
#pragma unroll
                        for (int kb = 0; kb < 2; ++kb) {
                            tma_load_4d(dst + kb * 16384, &tmV, bar(kBarVfull + s), kb * 64, k0, it.h, it.b);
                            tma_load_4d(dst + kb * 16384 + 8192, &tmV, bar(kBarVfull + s), kb * 64, k1, it.h, it.b);
                        }
                    }
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar(kBarMapFree + par)) : "memory");
        }
        // after an abort: the copies this warp started land before the CTA releases its memory
        if (lane == 0 && *abort_flag) {
            auto drain = [&](uint32_t b, int issued) {
                if (issued == 0) return;
                for (long long it = 0; it < kWaitLimit; ++it)
                    if (mbar_try_wait(b, (uint32_t)(issued - 1) & 1u)) break;
            };
            drain(bar(kBarQfull), issuedQ);
            for (int s = 0; s < kStages; ++s) {  // uses of slot s among the first n ring entries
                drain(bar(kBarKfull + s), issuedK > s ? (issuedK - s + kStages - 1) / kStages : 0);
                drain(bar(kBarVfull + s), issuedV > s ? (issuedV - s + kStages - 1) / kStages : 0);
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issue
        const uint32_t idS = idesc_bf16(kM, 2 * kHalf, false);
        const uint32_t idPV = idesc_bf16(kM, kHead, true);
        auto issue_s = [&](int x, int s) {  // S_x = Q_x K_s^T
            const uint32_t d = tmem + x * 128;
#pragma unroll
            for (int ks = 0; ks < kHead / 16; ++ks) {
                const uint32_t qa = sbase + kQOff + x * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32;
                const uint32_t ka = sbase + kKOff + s * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_ss(d, smem_desc(qa, 16, 1024), smem_desc(ka, 16, 1024), idS, ks > 0);
            }
            mma_commit(bar(kBarSfull + x));
        };
        auto issue_pv = [&](int x, int s, bool acc) {  // O_x (+)= P_x V_s
#pragma unroll
            for (int ks = 0; ks < 2 * kHalf / 16; ++ks) {
                const uint32_t va = sbase + kVOff + s * 32768 + ks * 2048;
                mma_ts(tmem + 256 + x * 128, tmem + x * 128 + ks * 8, smem_desc(va, 16384, 1024), idPV,
                       (acc || ks > 0) ? 1u : 0u);
            }
            mma_commit(bar(kBarOdone + x));
        };
        int g = 0, qn = 0;
        bool ok = true;
        for (int r = 0, n = 0; ok; ++r, ++n) {
            const int j = item_of(r, cta, G);
            if (j >= args.items) break;
            const Item it = decode_item(args, j);
            const int par = n & 1;
            if (!(ok = wait_warp(bar(kBarMapReady + par), (n >> 1) & 1))) break;
            const int nu = (int)union_count[par];
            const int nt = it.nwt + ((nu + 1) >> 1);
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar(kBarMapFree + par)) : "memory");
            if (nt == 0) continue;
            if (!(ok = wait_warp(bar(kBarQfull), qn & 1))) break;
            ++qn;
            tc_fence_after();
            for (int i = 0; i < nt; ++i, ++g) {
                const int s = g % kStages, u = g / kStages;
                if (!(ok = wait_warp(bar(kBarKfull + s), u & 1))) break;
                tc_fence_after();
                if (lane == 0) issue_s(0, s);
                if (i > 0) {  // PV_B of the previous tile
                    if (!(ok = wait_warp(bar(kBarPfull + 1), (g - 1) & 1))) break;
                    tc_fence_after();
                    if (lane == 0) {
                        issue_pv(1, (g - 1) % kStages, i > 1);
                        mma_commit(bar(kBarVfree + (g - 1) % kStages));
                    }
                }
                if (lane == 0) {
                    issue_s(1, s);
                    mma_commit(bar(kBarKfree + s));
                    if (i == nt - 1) mma_commit(bar(kBarQfree));
                }
                if (!(ok = wait_warp(bar(kBarPfull + 0), g & 1))) break;
                if (!(ok = wait_warp(bar(kBarVfull + s), u & 1))) break;
                tc_fence_after();
                if (lane == 0) issue_pv(0, s, i > 0);
                __syncwarp();
            }
            if (!ok) break;
            if (!(ok = wait_warp(bar(kBarPfull + 1), (g - 1) & 1))) break;
            tc_fence_after();
            if (lane == 0) {
                issue_pv(1, (g - 1) % kStages, nt > 1);
                mma_commit(bar(kBarVfree + (g - 1) % kStages));
            }
            __syncwarp();
        }
        // every MMA this warp issued completes before TMEM and shared memory are released
        if (lane == 0) {
            mma_commit(bar(kBarDrain));
            for (long long it = 0; it < kWaitLimit; ++it)
                if (mbar_try_wait(bar(kBarDrain), 0)) break;
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax rows
        const int x = warp >> 2;            // query tile A (0) or B (1)
        const int quad = warp & 3;          // TMEM lane quadrant
        const int rloc = quad * 32 + lane;  // row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const uint32_t s_col = tmem + lane_base + x * 128;
        const uint32_t o_col = tmem + lane_base + 256 + x * 128;
        int g = 0;  // tiles processed by this query tile, over all items
        for (int r = 0, n = 0;; ++r, ++n) {
            const int j = item_of(r, cta, G);
            if (j >= args.items) break;
            const Item it = decode_item(args, j);
            const int par = n & 1;
            const int t = it.t0 + x * kM + rloc;
            const bool row_ok = t < args.N;
            const int64_t qrow = ((int64_t)it.b * a.H + it.h) * a.Lq + t;
            const int nsel = (row_ok && a.topk > 0) ? min(max(__ldg(&a.nsel[qrow]), 0), a.topk) : 0;
            const int32_t *ip = a.idx + qrow * a.topk;
            const float *sp = a.score + qrow * a.topk;
            float ref = -INFINITY;  // log2-domain reference: the largest kept chunk score
            for (int k = 0; k < nsel; ++k) {
                const int c = __ldg(&ip[k]);
                if (c >= 0 && c < args.C) ref = fmaxf(ref, __ldg(&sp[k]) * kLog2e);
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
            const int nu = (int)union_count[par];
            const int nt = it.nwt + ((nu + 1) >> 1);
            const uint32_t *bm = bitmaps + par * kMaxBitmapWords;
            float m_used = ref;
            float l = 0.f;
            int cur = -1;
            bool ok = true;
            for (int i = 0; i < nt; ++i, ++g) {
                if (!(ok = wait_warp(bar(kBarSfull + x), g & 1))) break;
                tc_fence_after();
                uint32_t sr[64];
                uint32_t pk[32];
                if (i < it.nwt) {
                    // ---- window tile: halves at ks0, ks1 (the second may be empty)
                    const int ks0 = it.ws0 + kHalf * (2 * i);
                    const bool h1 = 2 * i + 1 < it.nhw;
                    const int ks1 = ks0 + kHalf;
                    // valid key offsets j in [jlo, jhi] of each half for this row
                    auto range = [&](int ks, bool valid, int &jlo, int &jhi) {
                        jlo = max(0, t - a.W + 1 - ks);
                        jhi = min(kHalf - 1, t - ks);
                        if (!valid || !row_ok) {
                            jlo = kHalf;
                            jhi = -1;
                        }
                    };
                    int lo0, hi0, lo1, hi1;
                    range(ks0, true, lo0, hi0);
                    range(ks1, h1, lo1, hi1);
                    const bool full0 = __all_sync(kFull, lo0 == 0 && hi0 == kHalf - 1);
                    const bool full1 = __all_sync(kFull, lo1 == 0 && hi1 == kHalf - 1);
                    const bool none1 = __all_sync(kFull, lo1 > hi1);
                    auto half_max = [&](bool full, int jlo, int jhi) {
                        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
                        if (full) {
#pragma unroll
                            for (int q = 0; q < 64; q += 8) {
                                m0 = max3(m0, __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]));
                                m1 = max3(m1, __uint_as_float(sr[q + 2]), __uint_as_float(sr[q + 3]));
                                m2 = max3(m2, __uint_as_float(sr[q + 4]), __uint_as_float(sr[q + 5]));
                                m3 = max3(m3, __uint_as_float(sr[q + 6]), __uint_as_float(sr[q + 7]));
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 64; ++q) {
                                const bool v = q >= jlo && q <= jhi;
                                sr[q] = v ? sr[q] : __float_as_uint(-INFINITY);
                            }
#pragma unroll
                            for (int q = 0; q < 64; q += 8) {
                                m0 = max3(m0, __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]));
                                m1 = max3(m1, __uint_as_float(sr[q + 2]), __uint_as_float(sr[q + 3]));
                                m2 = max3(m2, __uint_as_float(sr[q + 4]), __uint_as_float(sr[q + 5]));
                                m3 = max3(m3, __uint_as_float(sr[q + 6]), __uint_as_float(sr[q + 7]));
                            }
                        }
                        return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
                    };
                    float mt = -INFINITY;
                    if (!none1) {
                        tmem_ld32(s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                        tmem_ld32(s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                        tmem_wait_ld();
                        mt = half_max(full1, lo1, hi1);
                    }
                    tmem_ld32(s_col, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                    tmem_wait_ld();
                    mt = fmaxf(mt, half_max(full0, lo0, hi0)) * scale2;
                    // raise the row's reference when its tile max passes it by more than 8
                    const bool raise = mt != -INFINITY && (m_used == -INFINITY || mt > m_used + 8.f);
                    const float f = raise ? ex2(m_used - mt) : 1.f;  // 0 when m_used is -inf
                    if (__any_sync(kFull, raise && l > 0.f)) {
                        // O holds earlier tiles of this item: PV_x of the previous tile completes first
                        if (!(ok = wait_warp(bar(kBarOdone + x), (g - 1) & 1))) break;
                        tc_fence_after();
#pragma unroll
                        for (int part = 0; part < 4; ++part) {
                            uint32_t o[32];
                            tmem_ld32(o_col + part * 32, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * f);
                            tmem_st32(o_col + part * 32, o);
                        }
                    }
                    if (raise) {
                        l *= f;
                        m_used = mt;
                    }
                    const float nb = m_used == -INFINITY ? 0.f : -m_used;
                    auto half_exp = [&]() {  // sr (masked) -> pk, returns the sum
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
                            pk[q >> 1] = pack_bf16(e0, e1);
                            pk[(q >> 1) + 1] = pack_bf16(e2, e3);
                        }
                        return (z0 + z1) + (z2 + z3);
                    };
                    // half 0 (still in registers, masked) -> P columns [0, 32)
                    l += half_exp();
                    tmem_st32(s_col, pk);
                    // half 1 -> P columns [32, 64)
                    if (none1) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) pk[q] = 0u;
                    } else {
                        tmem_ld32(s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                        tmem_ld32(s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                        tmem_wait_ld();
                        if (!full1) {
#pragma unroll
                            for (int q = 0; q < 64; ++q) {
                                const bool v = q >= lo1 && q <= hi1;
                                sr[q] = v ? sr[q] : __float_as_uint(-INFINITY);
                            }
                        }
                        l += half_exp();
                    }
                    tmem_st32(s_col + 32, pk);
                } else {
                    // ---- chunk tile: two union chunks (the second may be empty)
                    const int c0 = next_bit(bm, nwords, cur + 1);
                    const int c1 = next_bit(bm, nwords, c0 + 1);
                    cur = c1 >= 0 ? c1 : c0;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int c = hh == 0 ? c0 : c1;
                        const bool sel = row_ok && c >= 0 && qc[0] == c;
                        float wgt = 0.f;
                        if (sel) {
                            wgt = ex2(qs[0] - m_used);
                            l += wgt;
                            qc[0] = qc[1];
                            qs[0] = qs[1];
                            qc[1] = qc[2];
                            qs[1] = qs[2];
                            qc[2] = qc[3];
                            qs[2] = qs[3];
                            qc[3] = kn < nsel ? __ldg(&ip[kn]) : INT_MAX;
                            qs[3] = kn < nsel ? __ldg(&sp[kn]) * kLog2e : 0.f;
                            ++kn;
                        }
                        if (__any_sync(kFull, sel)) {
                            tmem_ld32(s_col + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                            tmem_ld32(s_col + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                            tmem_wait_ld();
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
                            const float z = (z0 + z1) + (z2 + z3);
                            const float fw = sel ? __fdividef(wgt, z) : 0.f;  // z >= 1: the max term is 1
#pragma unroll
                            for (int q = 0; q < 32; ++q)
                                pk[q] = pack_bf16(__uint_as_float(sr[2 * q]) * fw, __uint_as_float(sr[2 * q + 1]) * fw);
                        } else {
#pragma unroll
                            for (int q = 0; q < 32; ++q) pk[q] = 0u;
                        }
                        tmem_st32(s_col + hh * 32, pk);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar(kBarPfull + x)) : "memory");
            }
            // ---- epilogue: O / l and lse
            if (ok && nt > 0) ok = wait_warp(bar(kBarOdone + x), (g - 1) & 1);
            if (!ok) break;
            tc_fence_after();
            bf16 *orow = static_cast<bf16 *>(a.O.ptr) + it.b * a.O.sb + it.h * a.O.sh + (int64_t)t * a.O.st;
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
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar(kBarMapFree + par)) : "memory");
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
    if (!make_map(&mq, a.Q, a.B, a.H, N, kM) || !make_map(&mk, a.K, a.B, a.H, N, kHalf) ||
        !make_map(&mv, a.V, a.B, a.H, N, kHalf))
        return HILS_ERR_CUDA;
    static KernelSetup setup;
    int per_sm = 0;
    const hils_status st = kernel_setup(setup, (const void *)attend_prefill_tc_kernel, kThreads, kSmemBytes, &per_sm);
    if (st != HILS_OK) return st;
    if (per_sm < 1) return HILS_ERR_CUDA;
    TcArgs ta;
    ta.a = a;
    ta.N = N;
    ta.C = N / kChunk;
    ta.nqb = (N + kRows - 1) / kRows;
    ta.items = a.B * a.H * ta.nqb;
    ta.status = status;
    const int grid = min(ta.items, per_sm * device_sm_count());
    attend_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, ta);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace hils
