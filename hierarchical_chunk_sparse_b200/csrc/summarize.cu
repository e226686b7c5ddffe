// Landmark chunk summaries: "Hierarchical Sparse Attention Done Right" (picx.dev
// summary), Methodology 1, Eq. 8.
//
// For chunk c of head (b, h):  l_j = scale * q'_c . k_j (S = 64 keys),  p = softmax(l),
//   k'_c = sum_j p_j k_j,  b'_c = -sum_j p_j log p_j.
// The entropy is evaluated as sum_j p_j (log Z - (l_j - m)) with m = max l and
// Z = sum_j exp(l_j - m): the same quantity, written as a sum of non-negative terms.
//
// Design: the pass is bound by HBM bandwidth (it reads every key once, about one
// flop per byte). A persistent grid of 128-thread CTAs walks the chunks; each chunk
// (64 key rows plus its landmark row) is copied into shared memory with 16-byte
// cp.async copies, three chunks in flight per CTA. Logits use two threads per key
// row; the landmark softmax runs in one warp; the weighted key sum gives each
// thread two adjacent columns over a quarter or half of the rows.
//
// Decode-time (incremental) form, with cache_len: one unit per (b, h); the unit is the
// chunk that sequence b's newest token completed (cache_len[b] a positive multiple of
// 64), or nothing. The same per-chunk arithmetic writes the same bits as the full pass.
#include "hils_internal.cuh"

namespace hils {
namespace {

template <typename T, int D>
struct SumCfg {
    static constexpr int kThreads = 128;
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kRowUnits = kRowBytes / 16;          // 16-byte units per row
    static constexpr int kHalfUnits = kRowUnits / 2;          // units per half row (4, 8 or 16)
    static constexpr int kStageUnits = (kChunk + 1) * kRowUnits;
    static constexpr int kStageBytes = kStageUnits * 16;
    static constexpr int kStages = 3;
    static constexpr int kColUnits = D / 2;                   // two columns per thread
    static constexpr int kRowGroups = kThreads / kColUnits;   // 2 (d=128) or 4 (d=64)
    static constexpr int kSmemBytes = kStages * kStageBytes + (2 * kChunk + kRowGroups * D) * 4;
    static_assert(kHalfUnits == 4 || kHalfUnits == 8 || kHalfUnits == 16, "row size");
};

// Order in which a thread walks the 16-byte units of its half row: rotated so that
// the 8 threads of a shared-memory phase (4 rows x 2 halves) hit 8 distinct bank groups.
template <int kHalfUnits>
__device__ __forceinline__ int rotated_unit(int k, int row, int half) {
    if (kHalfUnits == 4) return (k + row) & 3;
    return (k + 2 * row + half) & (kHalfUnits - 1);
}

template <typename T, int D>
__global__ void __launch_bounds__(128) summarize_kernel(SummarizeArgs a) {
    using Cfg = SumCfg<T, D>;
    extern __shared__ __align__(16) uint8_t smem[];
    float *logit = reinterpret_cast<float *>(smem + Cfg::kStages * Cfg::kStageBytes);
    float *prob = logit + kChunk;
    float *red = prob + kChunk;

    const int tid = threadIdx.x;
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

    auto issue = [&](unsigned u, int stage) {
        int c = -1, bh = 0;
        if (u < total) unit_chunk(u, bh, c);
        if (c >= 0) {
            const int h = bh % a.H;
            const int b = bh / a.H;
            const T *k0 = static_cast<const T *>(a.K.ptr) + b * a.K.sb + (h / a.G) * a.K.sh +
                          (int64_t)c * kChunk * a.K.st;  // the query head's key-value head
            const T *lq = static_cast<const T *>(a.LQ.ptr) + b * a.LQ.sb + h * a.LQ.sh + c * a.LQ.st;
            uint8_t *dst = smem + stage * Cfg::kStageBytes;
            for (int i = tid; i < Cfg::kStageUnits; i += Cfg::kThreads) {
                const int row = i / Cfg::kRowUnits, un = i % Cfg::kRowUnits;
                const T *src = row < kChunk ? k0 + row * a.K.st : lq;
                cp_async16(dst + i * 16, reinterpret_cast<const uint8_t *>(src) + un * 16);
            }
        }
        cp_async_commit();
    };

#pragma unroll
    for (int s = 0; s < Cfg::kStages - 1; ++s) issue(blockIdx.x + s * stride, s);

    int stage = 0;
    for (unsigned u = blockIdx.x; u < total; u += stride) {
        issue(u + (Cfg::kStages - 1) * stride, (stage + Cfg::kStages - 1) % Cfg::kStages);
        cp_async_wait<Cfg::kStages - 1>();
        __syncthreads();

        const uint8_t *tile = smem + stage * Cfg::kStageBytes;
        int ubh, uc;
        unit_chunk(u, ubh, uc);
        if (uc >= 0) {  // uniform over the CTA
        // landmark logits, two threads per key row
        {
            const int row = tid >> 1, half = tid & 1;
            const uint4 *krow = reinterpret_cast<const uint4 *>(tile + row * Cfg::kRowBytes);
            const uint4 *lrow = reinterpret_cast<const uint4 *>(tile + kChunk * Cfg::kRowBytes);
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < Cfg::kHalfUnits; ++k) {
                const int un = half * Cfg::kHalfUnits + rotated_unit<Cfg::kHalfUnits>(k, row, half);
                acc = dot16<T>(krow[un], lrow[un], acc);
            }
            acc += __shfl_xor_sync(kFull, acc, 1);
            if (half == 0) logit[row] = acc * a.scale;
        }
        __syncthreads();
        // softmax and entropy in warp 0
        if (tid < 32) {
            const float l0 = logit[tid], l1 = logit[tid + 32];
            const float m = warp_max(fmaxf(l0, l1));
            const float e0 = expf(l0 - m), e1 = expf(l1 - m);
            const float z = warp_sum(e0 + e1);
            const float inv = 1.f / z, lz = logf(z);
            const float p0 = e0 * inv, p1 = e1 * inv;
            prob[tid] = p0;
            prob[tid + 32] = p1;
            const float ent = warp_sum(p0 * (lz - (l0 - m)) + p1 * (lz - (l1 - m)));
            if (tid == 0) a.Bsum[(int64_t)ubh * a.C + uc] = ent;
        }
        __syncthreads();
        // k'_c = sum_j p_j k_j: thread owns columns 2*cu, 2*cu+1 over rows rg, rg+G, ...
        {
            const int cu = tid % Cfg::kColUnits, rg = tid / Cfg::kColUnits;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
            for (int j = rg; j < kChunk; j += Cfg::kRowGroups) {
                const float2 kv = load2(reinterpret_cast<const T *>(tile + j * Cfg::kRowBytes) + 2 * cu);
                const float pj = prob[j];
                a0 = fmaf(pj, kv.x, a0);
                a1 = fmaf(pj, kv.y, a1);
            }
            red[rg * D + 2 * cu] = a0;
            red[rg * D + 2 * cu + 1] = a1;
            __syncthreads();
            if (rg == 0) {
#pragma unroll
                for (int g = 1; g < Cfg::kRowGroups; ++g) {
                    a0 += red[g * D + 2 * cu];
                    a1 += red[g * D + 2 * cu + 1];
                }
                const int h = ubh % a.H;
                const int b = ubh / a.H;
                T *out = static_cast<T *>(a.Ksum.ptr) + b * a.Ksum.sb + h * a.Ksum.sh + uc * a.Ksum.st;
                store2(out + 2 * cu, a0, a1);
            }
        }
        }
        __syncthreads();
        stage = (stage + 1) % Cfg::kStages;
    }
    cp_async_wait<0>();
}

template <typename T, int D>
hils_status launch(const SummarizeArgs &a, cudaStream_t s) {
    using Cfg = SumCfg<T, D>;
    const int64_t total = a.cache_len ? (int64_t)a.B * a.H : (int64_t)a.B * a.H * a.C;
    if (total == 0 || a.C == 0) return HILS_OK;
    static KernelSetup setup;
    int per_sm = 1;
    const hils_status st = kernel_setup(setup, (const void *)summarize_kernel<T, D>, Cfg::kThreads,
                                        Cfg::kSmemBytes, &per_sm);
    if (st != HILS_OK) return st;
    const int64_t grid = total < (int64_t)per_sm * device_sm_count() ? total
                                                                      : (int64_t)per_sm * device_sm_count();
    summarize_kernel<T, D><<<(unsigned)grid, Cfg::kThreads, Cfg::kSmemBytes, s>>>(a);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace

hils_status launch_summarize(hils_dtype dt, int d, const SummarizeArgs &a, cudaStream_t s) {
    if (dt == HILS_BF16) return d == 64 ? launch<bf16, 64>(a, s) : launch<bf16, 128>(a, s);
    return d == 64 ? launch<float, 64>(a, s) : launch<float, 128>(a, s);
}

}  // namespace hils
