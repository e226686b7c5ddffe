// Landmark chunk summaries: "Hierarchical Sparse Attention Done Right" (picx.dev
// summary), Methodology 1, Eq. 8.
//
// For chunk c of head (b, h):  l_j = scale * q'_c . k_j (S = 64 keys),  p = softmax(l),
//   k'_c = sum_j p_j k_j,  b'_c = -sum_j p_j log p_j.
// With m = max l and z = sum_j exp(l_j - m), the entropy is
//   b'_c = log z - (1/z) sum_j exp(l_j - m) (l_j - m),
// the same quantity written through the softmax's own sums.
//
// Design: the pass is bound by HBM bandwidth (it reads every key once, about one flop
// per byte). A persistent grid of CTAs walks the chunks. In each CTA a producer warp
// fills a ring of stages with bulk copies (the chunk's 64 key rows, one copy when the
// rows are contiguous, else one per row; and its landmark row), each completing on the
// stage's mbarrier, while four compute warps take 16 key rows each: two lanes per row
// form the landmark logits, the warp keeps its own maximum, sum and entropy sum, and
// each lane accumulates D/32 columns of its rows' exp-weighted keys. One exchange
// through shared memory combines the four warps (rescaled to the chunk maximum) into
// k'_c and b'_c, and the stage is handed back to the producer.
//
// Decode-time (incremental) form, with cache_len: one unit per (b, h); the unit is the
// chunk that sequence b's newest token completed (cache_len[b] a positive multiple of
// 64), or nothing. The same per-chunk arithmetic writes the same bits as the full pass.
#include "tc_common.cuh"

namespace hils {
namespace {

constexpr int kSumWarps = 4;                   // compute warps, 16 key rows each
constexpr int kSumThreads = (kSumWarps + 1) * 32;  // + the producer warp
constexpr long long kSumWaitNs = 100ll * 1000 * 1000;  // bound of every wait on a copy or a release

template <typename T, int D>
struct SumCfg {
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kRowUnits = kRowBytes / 16;          // 16-byte units per row
    static constexpr int kHalfUnits = kRowUnits / 2;          // units per half row (4, 8 or 16)
    static constexpr int kStageBytes = (kChunk + 1) * kRowBytes;  // 64 key rows + the landmark row
    static constexpr int kStages = kStageBytes > 10000 ? 3 : 6;  // bf16, d = 128: 4 CTAs per SM
    static constexpr int kCols = D / 32;                      // columns per lane
    // per warp: max, sum, entropy sum, then the D exp-weighted column sums
    static constexpr int kXchgFloats = 4 + D;
    static constexpr int kSmemBytes = kStages * kStageBytes + kSumWarps * kXchgFloats * 4;
    static_assert(kHalfUnits == 4 || kHalfUnits == 8 || kHalfUnits == 16, "row size");
    static_assert(kStageBytes % 16 == 0, "bulk copy alignment");
};

// Order in which a lane walks the 16-byte units of its half row: rotated so that the
// lanes of a shared-memory phase (4 rows x 2 halves) hit distinct bank groups.
template <int kHalfUnits>
__device__ __forceinline__ int rotated_unit(int k, int row, int half) {
    if (kHalfUnits == 4) return (k + row) & 3;
    return (k + 2 * row + half) & (kHalfUnits - 1);
}

__device__ __forceinline__ uint64_t sum_global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void sum_bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void sum_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// Bounded wait on an mbarrier phase; false if the limit passed first.
__device__ __forceinline__ bool sum_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = sum_global_ns();
    for (int it = 0;; ++it) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 15 && sum_global_ns() - t0 > (uint64_t)kSumWaitNs) return false;
    }
}

// The j-th element pair (columns 2j, 2j+1) of a row, as floats.
__device__ __forceinline__ float2 pair_at(const bf16 *row, int j) { return load2(row + 2 * j); }
__device__ __forceinline__ float2 pair_at(const float *row, int j) { return load2(row + 2 * j); }

template <typename T, int D>
__global__ void __launch_bounds__(kSumThreads) summarize_kernel(SummarizeArgs a) {
    using Cfg = SumCfg<T, D>;
    constexpr int kStages = Cfg::kStages;
    extern __shared__ __align__(16) uint8_t smem[];
    float *xchg = reinterpret_cast<float *>(smem + kStages * Cfg::kStageBytes);
    __shared__ unsigned long long full_bar[kStages], empty_bar[kStages];
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // units: every (b, h, chunk), or with cache_len one per (b, h)
    const unsigned total = a.cache_len ? (unsigned)a.B * a.H : (unsigned)a.B * a.H * a.C;  // checked to fit
    const unsigned stride = gridDim.x;
    // the unit's (b, h) and chunk; chunk -1: nothing to summarise
    auto unit_chunk = [&](unsigned u, int &bh, int &c) {
        if (a.cache_len) {
            bh = (int)u;
            const int L = a.cache_len[bh / a.H];
            c = (L >= kChunk && L % kChunk == 0 && L / kChunk <= a.C) ? L / kChunk - 1 : -1;
        } else {
            c = (int)(u % (unsigned)a.C);
            bh = (int)(u / (unsigned)a.C);
        }
    };
    if (tid == 0) {
        s_abort = 0;
        for (int k = 0; k < kStages; ++k) {
            tc::mbar_init(tc::smem_u32(&full_bar[k]), 1);
            tc::mbar_init(tc::smem_u32(&empty_bar[k]), kSumWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();

    if (warp == kSumWarps) {
        // ---------------------------------------------------------------- producer warp
        int n = 0;
        for (unsigned u = blockIdx.x; u < total; u += stride, ++n) {
            const int s = n % kStages;
            if (n >= kStages) {  // the compute warps released this stage's previous chunk
                bool ok = true;
                if (lane == 0) ok = sum_wait(tc::smem_u32(&empty_bar[s]), (uint32_t)(n / kStages - 1) & 1u);
                ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
                if (!ok || *(volatile int *)&s_abort) {
                    if (lane == 0) s_abort = 1;
                    break;
                }
            }
            int bh, c;
            unit_chunk(u, bh, c);
            const uint32_t fb = tc::smem_u32(&full_bar[s]);
            uint8_t *st = smem + s * Cfg::kStageBytes;
            if (c < 0) {
                if (lane == 0) sum_arrive(fb);  // nothing to copy
                continue;
            }
            const int h = bh % a.H, b = bh / a.H;
            const T *k0 = static_cast<const T *>(a.K.ptr) + b * a.K.sb + (h / a.G) * a.K.sh +
                          (int64_t)c * kChunk * a.K.st;  // the query head's key-value head
            const T *lq = static_cast<const T *>(a.LQ.ptr) + b * a.LQ.sb + h * a.LQ.sh + c * a.LQ.st;
            if (lane == 0) {
                tc::mbar_expect_tx(fb, (uint32_t)Cfg::kStageBytes);
                sum_bulk_load(tc::smem_u32(st + kChunk * Cfg::kRowBytes), lq, Cfg::kRowBytes, fb);
            }
            __syncwarp();
            if (a.K.st == D) {  // the chunk's rows are contiguous
                if (lane == 0) sum_bulk_load(tc::smem_u32(st), k0, kChunk * Cfg::kRowBytes, fb);
            } else {
                for (int r = lane; r < kChunk; r += 32)
                    sum_bulk_load(tc::smem_u32(st + r * Cfg::kRowBytes), k0 + (int64_t)r * a.K.st, Cfg::kRowBytes, fb);
            }
        }
        // every copy started lands before the CTA leaves (bounded)
        if (lane == 0) {
            for (int j = (n > kStages ? n - kStages : 0); j < n; ++j)
                sum_wait(tc::smem_u32(&full_bar[j % kStages]), (uint32_t)(j / kStages) & 1u);
        }
    } else {
        // ---------------------------------------------------------------- compute warps
        int n = 0;
        for (unsigned u = blockIdx.x; u < total; u += stride, ++n) {
            const int s = n % kStages;
            int bh, c;
            unit_chunk(u, bh, c);
            // a copy that never lands stops the CTA: the warps meet at the next barrier and
            // leave before writing anything
            if (!sum_wait(tc::smem_u32(&full_bar[s]), (uint32_t)(n / kStages) & 1u)) s_abort = 1;
            if (c >= 0) {
                const uint8_t *tile = smem + s * Cfg::kStageBytes;
                // landmark logits: rows 16w..16w+15, two lanes per row
                const int row = warp * 16 + (lane >> 1), half = lane & 1;
                const uint4 *krow = reinterpret_cast<const uint4 *>(tile + row * Cfg::kRowBytes);
                const uint4 *lrow = reinterpret_cast<const uint4 *>(tile + kChunk * Cfg::kRowBytes);
                float l = 0.f;
#pragma unroll
                for (int k = 0; k < Cfg::kHalfUnits; ++k) {
                    const int un = half * Cfg::kHalfUnits + rotated_unit<Cfg::kHalfUnits>(k, row, half);
                    l = dot16<T>(krow[un], lrow[un], l);
                }
                l += __shfl_xor_sync(kFull, l, 1);
                l *= a.scale;  // both lanes of the pair hold the row's logit
                // this warp's maximum, sum and entropy sum over its 16 rows
                float mw = l;
#pragma unroll
                for (int o = 16; o > 1; o >>= 1) mw = fmaxf(mw, __shfl_xor_sync(kFull, mw, o));
                const float e = expf(l - mw);
                float zw = half == 0 ? e : 0.f, hw = half == 0 ? e * (l - mw) : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    zw += __shfl_xor_sync(kFull, zw, o);
                    hw += __shfl_xor_sync(kFull, hw, o);
                }
                // exp-weighted key columns: lane owns columns [kCols*lane, kCols*(lane+1))
                float acc[Cfg::kCols];
#pragma unroll
                for (int x = 0; x < Cfg::kCols; ++x) acc[x] = 0.f;
#pragma unroll 4
                for (int j = 0; j < 16; ++j) {
                    const float ej = __shfl_sync(kFull, e, 2 * j);
                    const T *kr = reinterpret_cast<const T *>(tile + (warp * 16 + j) * Cfg::kRowBytes) +
                                  Cfg::kCols * lane;
#pragma unroll
                    for (int x = 0; x < Cfg::kCols / 2; ++x) {
                        const float2 kv = pair_at(kr, x);
                        acc[2 * x] = fmaf(ej, kv.x, acc[2 * x]);
                        acc[2 * x + 1] = fmaf(ej, kv.y, acc[2 * x + 1]);
                    }
                }
                float *mine = xchg + warp * Cfg::kXchgFloats;
                if (lane == 0) {
                    mine[0] = mw;
                    mine[1] = zw;
                    mine[2] = hw;
                }
#pragma unroll
                for (int x = 0; x < Cfg::kCols; ++x) mine[4 + Cfg::kCols * lane + x] = acc[x];
            }
            // the stage's rows are no longer read: hand it back; then combine the warps
            __syncwarp();
            if (lane == 0) sum_arrive(tc::smem_u32(&empty_bar[s]));
            asm volatile("bar.sync 1, %0;" ::"n"(kSumWarps * 32) : "memory");
            if (*(volatile int *)&s_abort) break;  // uniform: read after the barrier
            if (c >= 0) {
                float m = xchg[0];
#pragma unroll
                for (int w = 1; w < kSumWarps; ++w) m = fmaxf(m, xchg[w * Cfg::kXchgFloats]);
                float f[kSumWarps], z = 0.f, hs = 0.f;
#pragma unroll
                for (int w = 0; w < kSumWarps; ++w) {
                    const float mw = xchg[w * Cfg::kXchgFloats];
                    f[w] = expf(mw - m);
                    const float zw = xchg[w * Cfg::kXchgFloats + 1], hw = xchg[w * Cfg::kXchgFloats + 2];
                    z = fmaf(f[w], zw, z);
                    hs = fmaf(f[w], fmaf(mw - m, zw, hw), hs);
                }
                const float inv = 1.f / z;
                const int h = bh % a.H, b = bh / a.H;
                T *out = static_cast<T *>(a.Ksum.ptr) + b * a.Ksum.sb + h * a.Ksum.sh + (int64_t)c * a.Ksum.st;
                for (int p = tid; p < D / 2; p += kSumWarps * 32) {  // two adjacent columns per thread
                    float v0 = 0.f, v1 = 0.f;
#pragma unroll
                    for (int w = 0; w < kSumWarps; ++w) {
                        v0 = fmaf(f[w], xchg[w * Cfg::kXchgFloats + 4 + 2 * p], v0);
                        v1 = fmaf(f[w], xchg[w * Cfg::kXchgFloats + 4 + 2 * p + 1], v1);
                    }
                    store2(out + 2 * p, v0 * inv, v1 * inv);
                }
                if (tid == 0) a.Bsum[(int64_t)bh * a.C + c] = logf(z) - hs * inv;
            }
            // the exchange area is rewritten by the next chunk only after everyone read it
            asm volatile("bar.sync 1, %0;" ::"n"(kSumWarps * 32) : "memory");
        }
    }
}

template <typename T, int D>
hils_status launch(const SummarizeArgs &a, cudaStream_t s) {
    using Cfg = SumCfg<T, D>;
    const int64_t total = a.cache_len ? (int64_t)a.B * a.H : (int64_t)a.B * a.H * a.C;
    if (total == 0 || a.C == 0) return HILS_OK;
    static KernelSetup setup;
    int per_sm = 1;
    const hils_status st = kernel_setup(setup, (const void *)summarize_kernel<T, D>, kSumThreads,
                                        Cfg::kSmemBytes, &per_sm);
    if (st != HILS_OK) return st;
    const int64_t grid = total < (int64_t)per_sm * device_sm_count() ? total
                                                                      : (int64_t)per_sm * device_sm_count();
    summarize_kernel<T, D><<<(unsigned)grid, kSumThreads, Cfg::kSmemBytes, s>>>(a);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace

hils_status launch_summarize(hils_dtype dt, int d, const SummarizeArgs &a, cudaStream_t s) {
    if (dt == HILS_BF16) return d == 64 ? launch<bf16, 64>(a, s) : launch<bf16, 128>(a, s);
    return d == 64 ? launch<float, 64>(a, s) : launch<float, 128>(a, s);
}

}  // namespace hils
