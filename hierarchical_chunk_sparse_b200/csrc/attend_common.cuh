// Pieces of the decode attend shared by its kernels (attend.cu) and the fused decode
// step (decode_fused.cu): the plan of one unit of a query, the workspace layout of the
// units' partial results, and Eq. 10's combination of those partials ("Hierarchical
// Sparse Attention Done Right" (picx.dev summary), Methodology 2, Eq. 10):
//   o = sum_u exp(m_u) o_u / sum_u exp(m_u),  lse = log sum_u exp(m_u),
// where a chunk unit has m_u = s^_{i,c} (its select score) and o_u its own softmax-
// weighted values, and a window tile has m_u = log sum_j exp(scale q.k_j) over its tokens.
#pragma once
#include <math.h>

#include "hils_internal.cuh"

namespace hils {
namespace {

// Unit u of a query at position t: token range and log-mass source.
struct UnitPlan {
    int start, rows;  // rows == 0: empty unit
    bool is_chunk;
    float mass;       // chunk units: the select score
};

__device__ __forceinline__ UnitPlan plan_unit(int u, int t, int K, int W, const int32_t *idx_row,
                                              const float *score_row, int nsel) {
    UnitPlan p{0, 0, false, -INFINITY};
    if (t < 0) return p;
    if (u < K) {
        if (u >= nsel) return p;
        const int c = idx_row[u];
        if (c < 0) return p;
        const int start = c * kChunk;
        if (start > t) return p;
        p.start = start;
        p.rows = min(kChunk, t - start + 1);
        p.is_chunk = true;
        p.mass = score_row[u];
        return p;
    }
    const int w0 = max(0, t - W + 1);
    const int start = w0 + (u - K) * kChunk;
    if (W <= 0 || start > t) return p;
    p.start = start;
    p.rows = min(kChunk, t - start + 1);
    return p;
}

// plan_unit on already loaded inputs (the kept chunk index and score of unit u).
__device__ __forceinline__ UnitPlan plan_unit_loaded(int u, int t, int K, int W, int c, float score, int nsel) {
    UnitPlan p{0, 0, false, -INFINITY};
    if (t < 0) return p;
    if (u < K) {
        if (u >= nsel || c < 0) return p;
        const int start = c * kChunk;
        if (start > t) return p;
        p.start = start;
        p.rows = min(kChunk, t - start + 1);
        p.is_chunk = true;
        p.mass = score;
        return p;
    }
    const int w0 = max(0, t - W + 1);
    const int start = w0 + (u - K) * kChunk;
    if (W <= 0 || start > t) return p;
    p.start = start;
    p.rows = min(kChunk, t - start + 1);
    return p;
}

struct DecodeWs {
    int *counters;  // [queries] units arrived
    float *mass;
    float *vec;
};

__host__ __device__ __forceinline__ size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__device__ __forceinline__ DecodeWs decode_ws(void *ws, int queries, int units, int D) {
    DecodeWs w;
    uint8_t *p = static_cast<uint8_t *>(ws);
    w.counters = reinterpret_cast<int *>(p);
    p += attend_decode_counter_bytes(queries);
    w.mass = reinterpret_cast<float *>(p);
    p += align256((size_t)queries * units * sizeof(float));
    w.vec = reinterpret_cast<float *>(p);
    return w;
}

template <typename T, int D>
__device__ __forceinline__ void store_output(const AttendArgs &a, int b, int h, int i, int64_t qi,
                                             const float *o, float lse) {
    T *orow = static_cast<T *>(a.O.ptr) + b * a.O.sb + h * a.O.sh + i * a.O.st;
    for (int x2 = threadIdx.x; x2 < D / 2; x2 += blockDim.x) store2(orow + 2 * x2, o[2 * x2], o[2 * x2 + 1]);
    if (a.lse && threadIdx.x == 0) a.lse[qi] = lse;
}

// o = sum_u e^{m_u - M} o_u / sum_u e^{m_u - M} and lse = M + log(sum) over `units`
// partials (masses m_u, vectors o_u, written to global memory by other CTAs). Thread x
// owns column x; every 32 units it issues all their mass and column loads at once and
// folds them into a running (max, sum, weighted column) triple, so one round trip per
// 32 units. Writes o to out[0..D) and lse to out[D].
template <int D>
__device__ void combine_units(const float *mass, const float *vec, int units, float *out) {
    constexpr int kB = 32;
    const int x = threadIdx.x;
    float M = -INFINITY, z = 0.f, acc = 0.f;
    if (x < D) {
        for (int v0 = 0; v0 < units; v0 += kB) {
            float m[kB], c[kB];
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                const bool ok = v0 + k < units;
                m[k] = ok ? __ldcg(mass + v0 + k) : -INFINITY;
                c[k] = ok ? __ldcg(vec + (size_t)(v0 + k) * D + x) : 0.f;
            }
            float mb = M;
#pragma unroll
            for (int k = 0; k < kB; ++k) mb = fmaxf(mb, m[k]);
            if (mb == -INFINITY) continue;
            const float f = expf(M - mb);  // 0 when M is -inf
            z *= f;
            acc *= f;
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                const float wv = expf(m[k] - mb);
                z += wv;
                acc = fmaf(wv, c[k], acc);
            }
            M = mb;
        }
        out[x] = M == -INFINITY ? 0.f : acc / z;
        if (x == 0) out[D] = M == -INFINITY ? -INFINITY : M + logf(z);
    }
    __syncthreads();
}

}  // namespace
}  // namespace hils
