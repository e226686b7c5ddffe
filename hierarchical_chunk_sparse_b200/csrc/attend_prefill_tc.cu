// Prefill attend on the 5th-generation tensor cores (bf16, d = 128): "Hierarchical
// Sparse Attention Done Right" (picx.dev summary), Methodology 2, Eq. 10, and the
// rcap.io post's pseudocode figure.
//
// One CTA (128 threads, one query row per thread) takes a tile of 128 consecutive
// queries [t0, t0+128) of one (b, h) and walks 64-key tiles in this order:
//   1. the window tiles covering [max(0, t0-W+1), t0+127], with an online softmax
//      whose reference max is raised (and O rescaled) only when a row's max exceeds
//      it by more than 8 in log2 units;
//   2. the union of the chunks kept by the tile's 128 queries, ascending; a row that
//      kept chunk c weights the chunk's own softmax by exp(s^_c), a row that did not
//      contributes zero.
// Per tile: S = Q K^T (M=128, N=64, K=128: eight tcgen05.mma) into one of two 64-column
// TMEM buffers; each thread reads its row of S, writes its row of P (bf16) over the
// same TMEM columns; O += P V (M=128, N=128, K=64, A from TMEM) accumulates in a
// 128-column TMEM region. Q, K and V tiles arrive by TMA (128-byte swizzle, no
// multicast) on a two-slot ring per operand; thread 0 issues loads and MMAs, S of the
// next tile is issued before the softmax of the current one. The tensor pipe runs a
// CTA's tcgen05.mma in issue order, which is what lets S_{i+2} reuse the columns of
// P_i after PV_i. Every mbarrier wait is bounded: on expiry the CTA records an error
// in the status word, stops issuing work, drains what it issued, frees its TMEM and
// exits without writing outputs.
#include "tc_common.cuh"

namespace hils {
namespace {

using namespace tc;

constexpr int kM = 128;          // query rows per CTA
constexpr int kTileN = 64;       // keys per tile
constexpr int kHead = 128;       // head dimension
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 256;  // S0 [0,64), S1 [64,128), O [128,256)
constexpr uint32_t kOCol = 128;
constexpr int kMaxBitmapWords = 256; // union bitmap: up to 8192 chunks
constexpr long long kWaitLimit = 1ll << 26;

// shared memory map (offsets from the 1024-aligned base)
constexpr int kQOff = 0;                   // 2 blocks x [128 rows x 128 B]
constexpr int kKOff = 32768;               // 2 slots x 2 blocks x [64 x 128 B]
constexpr int kVOff = 65536;               // 2 slots x 2 blocks x [64 x 128 B]
constexpr int kBarOff = 98304;             // mbarriers
constexpr int kMiscOff = kBarOff + 128;    // tmem address, abort flag
constexpr int kBitmapOff = kMiscOff + 64;  // union bitmap
constexpr int kSmemBytes = kBitmapOff + kMaxBitmapWords * 4 + 1024;  // + alignment slack

enum { kBarQ = 0, kBarK = 1, kBarV = 3, kBarS = 5, kBarO = 7, kNumBars = 9 };

struct TcArgs {
    AttendArgs a;
    int N, C;
    uint32_t *status;  // nonzero after a wait expired
};

// smallest set bit >= from in the bitmap, or -1
__device__ __forceinline__ int next_bit(const uint32_t *bm, int nwords, int from) {
    int w = from >> 5;
    if (w >= nwords) return -1;
    uint32_t m = bm[w] & (0xffffffffu << (from & 31));
    while (true) {
        if (m) return (w << 5) + __ffs(m) - 1;
        if (++w >= nwords) return -1;
        m = bm[w];
    }
}

__global__ void __launch_bounds__(kThreads) attend_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                      const __grid_constant__ CUtensorMap tmK,
                                                                      const __grid_constant__ CUtensorMap tmV,
                                                                      TcArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const AttendArgs &a = args.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * kM;
    const int bh = blockIdx.y;
    const int b = bh / a.H, h = bh % a.H;
    const int N = args.N;
    const uint32_t sbase = smem_u32(smem);
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + kMiscOff);
    volatile uint32_t *abort_flag = misc + 1;
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + kBitmapOff);
    const int nwords = (args.C + 31) >> 5;
    auto bar = [&](int i) { return sbase + kBarOff + 8u * i; };

    // ---- set-up: barriers, TMEM, union bitmap
    for (int i = tid; i < nwords; i += kThreads) bitmap[i] = 0u;
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(sbase + kMiscOff),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    __syncthreads();
    // each row's kept chunks: bitmap of the union, and the row's reference max
    const int t = t0 + tid;
    const bool row_ok = t < N;
    const int64_t qrow = ((int64_t)b * a.H + h) * a.Lq + t;
    const int nsel = (row_ok && a.topk > 0) ? min(max(a.nsel[qrow], 0), a.topk) : 0;
    const float kLog2e = 1.4426950408889634f;
    float ref = -INFINITY;  // log2-domain reference of this row
    for (int k = 0; k < nsel; ++k) {
        const int c = a.idx[qrow * a.topk + k];
        if (c >= 0 && c < args.C) {
            atomicOr(&bitmap[c >> 5], 1u << (c & 31));
            ref = fmaxf(ref, a.score[qrow * a.topk + k] * kLog2e);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    // ---- tile sequence: window tiles, then the union of kept chunks
    int ws0 = 0, nw = 0;
    if (a.W > 0 && t0 < N) {
        const int lo = max(0, t0 - a.W + 1);
        const int hi = min(N - 1, t0 + kM - 1);
        ws0 = (lo / kTileN) * kTileN;
        nw = (hi - ws0) / kTileN + 1;
    }
    int nch = 0;
    for (int i = 0; i < nwords; ++i) nch += __popc(bitmap[i]);
    const int ntiles = nw + nch;

    // Cursor over the tile sequence: key start of tile i (window or chunk).
    struct Cursor {
        int i, chunk;  // chunk: last chunk index visited (for the union walk)
    };
    auto tile_start = [&](Cursor &cu) -> int {  // start of tile cu.i, advancing the chunk walk
        if (cu.i < nw) return ws0 + cu.i * kTileN;
        cu.chunk = next_bit(bitmap, nwords, cu.chunk + 1);
        return cu.chunk * kTileN;
    };

    // bounded waits; the first expiry aborts the CTA (every later wait returns at once)
    auto wait = [&](uint32_t barrier, uint32_t parity) {
        if (*abort_flag) return false;
        for (long long it = 0; it < kWaitLimit; ++it)
            if (mbar_try_wait(barrier, parity)) return true;
        *abort_flag = 1u;
        atomicOr(args.status, 1u);
        return false;
    };

    int issued[kNumBars] = {0, 0, 0, 0, 0, 0, 0, 0, 0};  // thread 0: completions it has started per barrier
    const uint32_t idS = idesc_bf16(kM, kTileN, false);
    const uint32_t idPV = idesc_bf16(kM, kHead, true);
    const int y_q = t0;
    // issuer-side cursors and state (thread 0 only)
    Cursor load_cur{0, -1};
    int load_start[2] = {0, 0};  // key start of the tile loaded in each slot
    auto load_k = [&](int slot, int start) {
        ++issued[kBarK + slot];
        mbar_expect_tx(bar(kBarK + slot), 2 * kTileN * 128);
        const uint32_t dst = sbase + kKOff + slot * 16384;
        tma_load_4d(dst, &tmK, bar(kBarK + slot), 0, start, h, b);
        tma_load_4d(dst + 8192, &tmK, bar(kBarK + slot), 64, start, h, b);
    };
    auto load_v = [&](int slot, int start) {
        ++issued[kBarV + slot];
        mbar_expect_tx(bar(kBarV + slot), 2 * kTileN * 128);
        const uint32_t dst = sbase + kVOff + slot * 16384;
        tma_load_4d(dst, &tmV, bar(kBarV + slot), 0, start, h, b);
        tma_load_4d(dst + 8192, &tmV, bar(kBarV + slot), 64, start, h, b);
    };
    auto issue_s = [&](int i) {  // S_i = Q K_i^T into S buffer i%2
        const int slot = i & 1;
        const uint32_t d = tmem + slot * 64;
#pragma unroll
        for (int ks = 0; ks < kHead / 16; ++ks) {
            const uint32_t qa = sbase + kQOff + (ks >> 2) * 16384 + (ks & 3) * 32;
            const uint32_t ka = sbase + kKOff + slot * 16384 + (ks >> 2) * 8192 + (ks & 3) * 32;
            mma_ss(d, smem_desc(qa, 16, 1024), smem_desc(ka, 16, 1024), idS, ks > 0);
        }
        ++issued[kBarS + slot];
        mma_commit(bar(kBarS + slot));
    };
    auto issue_pv = [&](int i) {  // O += P_i V_i, P_i in TMEM over S buffer i%2
        const int slot = i & 1;
#pragma unroll
        for (int ks = 0; ks < kTileN / 16; ++ks) {
            const uint32_t va = sbase + kVOff + slot * 16384 + ks * 2048;
            mma_ts(tmem + kOCol, tmem + slot * 64 + ks * 8, smem_desc(va, 8192, 1024), idPV, (i > 0 || ks > 0));
        }
        ++issued[kBarO + slot];
        mma_commit(bar(kBarO + slot));
    };

    if (tid == 0 && ntiles > 0) {
        ++issued[kBarQ];
        mbar_expect_tx(bar(kBarQ), 2 * kM * 128);
        tma_load_4d(sbase + kQOff, &tmQ, bar(kBarQ), 0, y_q, h, b);
        tma_load_4d(sbase + kQOff + 16384, &tmQ, bar(kBarQ), 64, y_q, h, b);
        for (int s = 0; s < 2 && s < ntiles; ++s) {
            load_start[s] = tile_start(load_cur);
            load_k(s, load_start[s]);
            load_v(s, load_start[s]);
            ++load_cur.i;
        }
        if (wait(bar(kBarQ), 0) && wait(bar(kBarK), 0)) issue_s(0);
    }

    // ---- main loop
    Cursor cur{0, -1};  // every thread walks the tile sequence
    float m_used = ref;  // log2-domain reference used for P
    float l = 0.f;
    const float scale2 = a.scale * kLog2e;
    int sel_k = 0;
    int sel_c = nsel > 0 ? a.idx[qrow * a.topk] : INT_MAX;
    float sel_s = nsel > 0 ? a.score[qrow * a.topk] * kLog2e : 0.f;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    for (int i = 0; i < ntiles; ++i) {
        const int start = tile_start(cur);
        ++cur.i;
        const bool window = i < nw;
        // (A) issue S of the next tile
        if (tid == 0 && i + 1 < ntiles) {
            if (wait(bar(kBarK + ((i + 1) & 1)), ((i + 1) >> 1) & 1)) issue_s(i + 1);
        }
        // (B) softmax of tile i
        wait(bar(kBarS + (i & 1)), (i >> 1) & 1);
        tc_fence_after();
        uint32_t sr[2][32];
        const uint32_t sbuf = tmem + lane_base + (i & 1) * 64;
        tmem_ld32(sbuf, sr[0]);
        tmem_ld32(sbuf + 32, sr[1]);
        tmem_wait_ld();
        float p[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) p[j] = __uint_as_float(sr[j >> 5][j & 31]) * scale2;
        if (window) {
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                const int key = start + j;
                const bool ok = row_ok && key <= t && key > t - a.W;
                p[j] = ok ? p[j] : -INFINITY;
                mt = fmaxf(mt, p[j]);
            }
            // raise the row's reference when its max passes it by more than 8 (log2 units)
            const bool raise = mt != -INFINITY && (m_used == -INFINITY || mt > m_used + 8.f);
            const float f = raise ? ex2(m_used - mt) : 1.f;  // 0 when m_used is -inf
            // O is rescaled by the whole warp (tcgen05.ld/st are warp-collective) if any
            // of its rows has accumulated something and raises its reference
            if (__any_sync(kFull, raise && l > 0.f)) {
                wait(bar(kBarO + ((i - 1) & 1)), ((i - 1) >> 1) & 1);  // PV_{i-1} has finished
                tc_fence_after();
#pragma unroll
                for (int part = 0; part < 4; ++part) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + kOCol + part * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                    tmem_st32(tmem + lane_base + kOCol + part * 32, o);
                }
                tmem_wait_st();
            }
            if (raise) {
                l *= f;
                m_used = mt;
            }
            float ls = 0.f;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                p[j] = p[j] == -INFINITY ? 0.f : ex2(p[j] - m_used);
                ls += p[j];
            }
            l += ls;
        } else {
            const int c = start / kTileN;
            const bool sel = row_ok && sel_c == c;
            if (sel) {
                float mc = -INFINITY;
#pragma unroll
                for (int j = 0; j < 64; ++j) mc = fmaxf(mc, p[j]);
                float z = 0.f;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    p[j] = ex2(p[j] - mc);
                    z += p[j];
                }
                const float wgt = ex2(sel_s - m_used);
                l += wgt;
                const float f = wgt / z;
#pragma unroll
                for (int j = 0; j < 64; ++j) p[j] *= f;
                ++sel_k;
                sel_c = sel_k < nsel ? a.idx[qrow * a.topk + sel_k] : INT_MAX;
                sel_s = sel_k < nsel ? a.score[qrow * a.topk + sel_k] * kLog2e : 0.f;
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) p[j] = 0.f;
            }
        }
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = pack_bf16(p[2 * j], p[2 * j + 1]);
        tmem_st32(sbuf, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        // (D) O += P_i V_i; then refill the slots this tile released
        if (tid == 0) {
            tc_fence_after();
            if (wait(bar(kBarV + (i & 1)), (i >> 1) & 1)) issue_pv(i);
            if (!*abort_flag && i + 2 < ntiles) {  // K slot i%2 is free: S_i has completed
                const int slot = i & 1;
                load_start[slot] = tile_start(load_cur);
                ++load_cur.i;
                load_k(slot, load_start[slot]);
            }
            // V slot (i+1)%2 held V_{i-1}: free once PV_{i-1} has completed
            if (i >= 1 && i + 1 < ntiles) {
                if (wait(bar(kBarO + ((i - 1) & 1)), ((i - 1) >> 1) & 1)) load_v((i + 1) & 1, load_start[(i + 1) & 1]);
            }
        }
    }

    // ---- epilogue: O / l, lse
    if (ntiles > 0) wait(bar(kBarO + ((ntiles - 1) & 1)), ((ntiles - 1) >> 1) & 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool ok = !*abort_flag;  // uniform: read after the barrier
    if (ok) {
        bf16 *orow = static_cast<bf16 *>(a.O.ptr) + b * a.O.sb + h * a.O.sh + (int64_t)t * a.O.st;
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int part = 0; part < 4; ++part) {
            uint32_t o[32];
            if (ntiles > 0) {  // uniform: every lane loads, rows past N are not stored
                tmem_ld32(tmem + lane_base + kOCol + part * 32, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] = 0u;
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
    } else if (tid == 0) {
        // a wait expired: every load and MMA this CTA started completes (bounded waits on
        // each barrier's last started phase) before its shared memory and TMEM are released
        for (int i = 0; i < kNumBars; ++i) {
            if (issued[i] == 0) continue;
            const uint32_t parity = (uint32_t)(issued[i] - 1) & 1u;
            for (long long it = 0; it < kWaitLimit; ++it)
                if (mbar_try_wait(bar(i), parity)) break;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
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
    if (!make_map(&mq, a.Q, a.B, a.H, N, kM) || !make_map(&mk, a.K, a.B, a.H, N, kTileN) ||
        !make_map(&mv, a.V, a.B, a.H, N, kTileN))
        return HILS_ERR_CUDA;
    static KernelSetup setup;
    const hils_status st = kernel_setup(setup, (const void *)attend_prefill_tc_kernel, kThreads, kSmemBytes, nullptr);
    if (st != HILS_OK) return st;
    TcArgs ta;
    ta.a = a;
    ta.N = N;
    ta.C = N / kChunk;
    ta.status = status;
    dim3 grid((N + kM - 1) / kM, a.B * a.H);
    attend_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, ta);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace hils
