// Hierarchical softmax over the selected chunks plus the sliding window:
// "Hierarchical Sparse Attention Done Right" (picx.dev summary), Methodology 2, Eq. 10
// (w_ij = exp(s_ij)/Z_{i,c(j)} * Z^_{i,c(j)}/Z^_i, with Z^_i normalising over the selected
// chunks and the window), and the rcap.io post's pseudocode figure.
//
// Both kernels here split the work of one query into "units" of at most 64 tokens:
//   - chunk unit (one kept chunk c): log-mass m_u = s^_{i,c} (the select score) and
//     o_u = sum_{j in c} softmax_j(scale q.k_j) v_j;
//   - window tile (64 consecutive tokens of [max(0,t-W+1), t]): log-mass
//     m_u = log sum_j exp(scale q.k_j) over the tile and o_u its softmax-weighted v.
// Eq. 10 is then  o = sum_u exp(m_u) o_u / sum_u exp(m_u),  lse = log sum_u exp(m_u):
// the window tiles together give exp(LSE_W) o_W, the chunks exp(s^_c) o_c.
//
// Decode (one query per (b, h), memory bound): one 128-thread CTA per unit streams the
// unit's K and V rows (16-byte cp.async into shared memory, K and V in flight
// together), writes (m_u, o_u) to the workspace, and the last CTA of the (b, h)
// combines them. The general prefill kernel (any dtype) gives one CTA per query and
// walks its units in turn with a running combination; the bf16 prefill fast path is
// a separate tensor-core kernel.
#include <math.h>

#include "attend_common.cuh"

namespace hils {
namespace {

constexpr int kThreads = 128;

template <typename T, int D>
struct UnitCfg {
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kRowUnits = kRowBytes / 16;
    static constexpr int kHalfUnits = kRowUnits / 2;
    static constexpr int kTileBytes = kChunk * kRowBytes;
    static constexpr int kColUnits = D / 2;
    static constexpr int kRowGroups = kThreads / kColUnits;
    // K tile, V tile, query row, logits, probabilities, column partial sums
    static constexpr int kSmemBytes = 2 * kTileBytes + kRowBytes + (2 * kChunk + kRowGroups * D) * 4;
};

template <int kHalfUnits>
__device__ __forceinline__ int rotated_unit(int k, int row, int half) {
    if (kHalfUnits == 4) return (k + row) & 3;
    return (k + 2 * row + half) & (kHalfUnits - 1);
}

struct UnitSmem {
    uint8_t *kt, *vt, *q;
    float *logit, *prob, *red;
};

template <typename T, int D>
__device__ __forceinline__ UnitSmem unit_smem(uint8_t *base) {
    using Cfg = UnitCfg<T, D>;
    UnitSmem s;
    s.kt = base;
    s.vt = base + Cfg::kTileBytes;
    s.q = base + 2 * Cfg::kTileBytes;
    s.logit = reinterpret_cast<float *>(s.q + Cfg::kRowBytes);
    s.prob = s.logit + kChunk;
    s.red = s.prob + kChunk;
    return s;
}

// Copies the query row and `rows` K rows (group 0), then `rows` V rows (group 1).
template <typename T, int D>
__device__ __forceinline__ void unit_issue(const UnitSmem &s, const T *qrow, const T *k0, int64_t kst,
                                           const T *v0, int64_t vst, int rows) {
    using Cfg = UnitCfg<T, D>;
    const int tid = threadIdx.x;
    for (int i = tid; i < rows * Cfg::kRowUnits; i += kThreads) {
        const int r = i / Cfg::kRowUnits, un = i % Cfg::kRowUnits;
        cp_async16(s.kt + i * 16, reinterpret_cast<const uint8_t *>(k0 + r * kst) + un * 16);
    }
    for (int i = tid; i < Cfg::kRowUnits; i += kThreads)
        cp_async16(s.q + i * 16, reinterpret_cast<const uint8_t *>(qrow) + i * 16);
    cp_async_commit();
    for (int i = tid; i < rows * Cfg::kRowUnits; i += kThreads) {
        const int r = i / Cfg::kRowUnits, un = i % Cfg::kRowUnits;
        cp_async16(s.vt + i * 16, reinterpret_cast<const uint8_t *>(v0 + r * vst) + un * 16);
    }
    cp_async_commit();
}

// Consumes the copies of unit_issue. Returns log sum_j exp(scale q.k_j) over the
// rows; leaves o_u = sum_j p_j v_j in s.red[0..D). All threads call it.
template <typename T, int D>
__device__ float unit_compute(const UnitSmem &s, int rows, float scale) {
    using Cfg = UnitCfg<T, D>;
    const int tid = threadIdx.x;
    cp_async_wait<1>();
    __syncthreads();
    {
        const int row = tid >> 1, half = tid & 1;
        const uint4 *krow = reinterpret_cast<const uint4 *>(s.kt + row * Cfg::kRowBytes);
        const uint4 *qv = reinterpret_cast<const uint4 *>(s.q);
        float acc = 0.f;
        if (row < rows) {
#pragma unroll
            for (int k = 0; k < Cfg::kHalfUnits; ++k) {
                const int un = half * Cfg::kHalfUnits + rotated_unit<Cfg::kHalfUnits>(k, row, half);
                acc = dot16<T>(krow[un], qv[un], acc);
            }
        }
        acc += __shfl_xor_sync(kFull, acc, 1);
        if (half == 0) s.logit[row] = row < rows ? acc * scale : -INFINITY;
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
        if (tid == 0) s.logit[0] = m + logf(z);  // row 0's logit is no longer needed
    }
    cp_async_wait<0>();
    __syncthreads();
    const float lse_tile = s.logit[0];
    {
        const int cu = tid % Cfg::kColUnits, rg = tid / Cfg::kColUnits;
        float a0 = 0.f, a1 = 0.f;
        for (int j = rg; j < rows; j += Cfg::kRowGroups) {
            const float2 vv = load2(reinterpret_cast<const T *>(s.vt + j * Cfg::kRowBytes) + 2 * cu);
            const float pj = s.prob[j];
            a0 = fmaf(pj, vv.x, a0);
            a1 = fmaf(pj, vv.y, a1);
        }
        s.red[rg * D + 2 * cu] = a0;
        s.red[rg * D + 2 * cu + 1] = a1;
        __syncthreads();
        if (rg == 0) {
#pragma unroll
            for (int g = 1; g < Cfg::kRowGroups; ++g) {
                a0 += s.red[g * D + 2 * cu];
                a1 += s.red[g * D + 2 * cu + 1];
            }
            s.red[2 * cu] = a0;
            s.red[2 * cu + 1] = a1;
        }
    }
    __syncthreads();
    return lse_tile;
}

// grid (units, B*H): one unit per CTA; the last CTA of each (b, h) combines.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) attend_decode_kernel(AttendArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int is_last;
    const UnitSmem s = unit_smem<T, D>(smem);
    const int u = blockIdx.x;
    const int64_t qi = blockIdx.y;  // (b, h), one query each
    const int b = (int)(qi / a.H), h = (int)(qi % a.H);
    const int hk = h / a.G;                                   // key-value head of h
    const int64_t qg = (int64_t)b * (a.H / a.G) + hk;         // the group's kept list
    const bool chunk_unit = u < a.topk;
    // dependent launch: chunk units wait for the preceding grid (the select's outputs
    // idx, score, nsel). Window tiles read only Q, K and V; they skip the wait only when
    // the caller guarantees that the preceding grid is this library's select, which
    // itself started after all earlier work on the stream (hils_decode).
    if (chunk_unit || !a.window_early) pdl_wait();
    pdl_trigger();  // a dependent-launched successor may be scheduled; it waits for this grid
    // the unit's small inputs, loaded together before anything depends on them
    const int clen = a.cache_len[b];
    const int ns = chunk_unit ? a.nsel[qg] : 0;
    const int cidx = chunk_unit ? a.idx[qg * a.topk + u] : -1;
    const float csc = chunk_unit ? a.score[qi * a.topk + u] : 0.f;
    const UnitPlan p = plan_unit_loaded(u, clen - 1, a.topk, a.W, cidx, csc, ns);
    const DecodeWs ws = decode_ws(a.ws, a.B * a.H, a.units, D);
    float *my_vec = ws.vec + ((size_t)qi * a.units + u) * D;
    if (p.rows > 0) {
        const T *qrow = static_cast<const T *>(a.Q.ptr) + b * a.Q.sb + h * a.Q.sh;
        const T *k0 = static_cast<const T *>(a.K.ptr) + b * a.K.sb + hk * a.K.sh + (int64_t)p.start * a.K.st;
        const T *v0 = static_cast<const T *>(a.V.ptr) + b * a.V.sb + hk * a.V.sh + (int64_t)p.start * a.V.st;
        unit_issue<T, D>(s, qrow, k0, a.K.st, v0, a.V.st, p.rows);
        const float lse_tile = unit_compute<T, D>(s, p.rows, a.scale);
        for (int x = threadIdx.x; x < D; x += kThreads) my_vec[x] = s.red[x];
        if (threadIdx.x == 0) ws.mass[qi * a.units + u] = p.is_chunk ? p.mass : lse_tile;
    } else {
        // an empty unit contributes weight 0; its vector is zeroed so that no stale value
        // can enter the combination
        for (int x = threadIdx.x; x < D; x += kThreads) my_vec[x] = 0.f;
        if (threadIdx.x == 0) ws.mass[qi * a.units + u] = -INFINITY;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(&ws.counters[qi], 1) == a.units - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    combine_units<D>(ws.mass + (size_t)qi * a.units, ws.vec + (size_t)qi * a.units * D, a.units, s.red);
    store_output<T, D>(a, b, h, 0, qi, s.red, s.red[D]);
    if (threadIdx.x == 0) ws.counters[qi] = 0;
}

// ---- grouped-query decode (summary page, Methodology 3, GQA adaptation): the GG query
// heads of a group read the same key-value head and keep the same chunks, so one CTA per
// (unit, b, group) copies the unit's K and V rows once and computes the unit for every
// head of the group (each head with its own query, softmax and chunk score); the
// group's last CTA combines every head's units.

template <typename T, int D, int GG>
struct GroupUnitCfg {
    using U = UnitCfg<T, D>;
    // K tile, V tile, the heads' query rows, logits and probabilities per head, column
    // partial sums per head
    static constexpr int kSmemBytes = 2 * U::kTileBytes + GG * U::kRowBytes +
                                      (2 * GG * kChunk + GG * U::kRowGroups * D) * 4;
};

// Eq. 10's combination for the GG heads of a group at once: kThreads / GG threads per
// head, D / (kThreads / GG) consecutive columns per thread, every load of a batch of
// units in flight together. mass and vec hold the heads' partials one after another
// (units per head). Writes head hh's o to out[hh * (D + 1) ..] and its lse after it.
template <int D, int GG>
__device__ void combine_group(const float *mass, const float *vec, int units, float *out) {
    constexpr int kTph = kThreads / GG, kCpt = D / kTph;
    constexpr int kB = kCpt >= 8 ? 8 : kCpt == 4 ? 16 : 32;
    static_assert(kCpt >= 1 && kTph * kCpt == D, "columns per thread");
    const int hh = threadIdx.x / kTph, x0 = (threadIdx.x % kTph) * kCpt;
    const float *mh = mass + (size_t)hh * units;
    const float *vh = vec + (size_t)hh * units * D + x0;
    float M = -INFINITY, z = 0.f, acc[kCpt];
#pragma unroll
    for (int q = 0; q < kCpt; ++q) acc[q] = 0.f;
    for (int v0 = 0; v0 < units; v0 += kB) {
        float m[kB], c[kB][kCpt];
#pragma unroll
        for (int k = 0; k < kB; ++k) {
            const bool ok = v0 + k < units;
            m[k] = ok ? __ldcg(mh + v0 + k) : -INFINITY;
#pragma unroll
            for (int q = 0; q < kCpt; ++q) c[k][q] = ok ? __ldcg(vh + (size_t)(v0 + k) * D + q) : 0.f;
        }
        float mb = M;
#pragma unroll
        for (int k = 0; k < kB; ++k) mb = fmaxf(mb, m[k]);
        if (mb == -INFINITY) continue;
        const float f = expf(M - mb);  // 0 when M is -inf
        z *= f;
#pragma unroll
        for (int q = 0; q < kCpt; ++q) acc[q] *= f;
#pragma unroll
        for (int k = 0; k < kB; ++k) {
            const float wv = expf(m[k] - mb);
            z += wv;
#pragma unroll
            for (int q = 0; q < kCpt; ++q) acc[q] = fmaf(wv, c[k][q], acc[q]);
        }
        M = mb;
    }
    float *oh = out + hh * (D + 1);
#pragma unroll
    for (int q = 0; q < kCpt; ++q) oh[x0 + q] = M == -INFINITY ? 0.f : acc[q] / z;
    if (x0 == 0) oh[D] = M == -INFINITY ? -INFINITY : M + logf(z);
    __syncthreads();
}

// grid (units, B * H / GG): one unit of one (b, group) per CTA.
template <typename T, int D, int GG>
__global__ void __launch_bounds__(kThreads) attend_decode_group_kernel(AttendArgs a) {
    using Cfg = UnitCfg<T, D>;
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int is_last;
    __shared__ float lse_h[GG];
    uint8_t *kt = smem, *vt = smem + Cfg::kTileBytes, *qsm = smem + 2 * Cfg::kTileBytes;
    float *logit = reinterpret_cast<float *>(qsm + GG * Cfg::kRowBytes);  // [GG][64]
    float *prob = logit + GG * kChunk;                                   // [GG][64]
    float *red = prob + GG * kChunk;                                     // [GG][kRowGroups][D]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int u = blockIdx.x;
    const int Hk = a.H / GG;
    const int64_t qg = blockIdx.y;  // (b, group): the group's kept list
    const int b = (int)(qg / Hk), hk = (int)(qg % Hk), h0 = hk * GG;
    const int64_t qi0 = (int64_t)b * a.H + h0;  // the group's first query head
    const bool chunk_unit = u < a.topk;
    if (chunk_unit || !a.window_early) pdl_wait();  // as in the per-head kernel
    pdl_trigger();
    const int clen = a.cache_len[b];
    const int ns = chunk_unit ? a.nsel[qg] : 0;
    const int cidx = chunk_unit ? a.idx[qg * a.topk + u] : -1;
    const UnitPlan p = plan_unit_loaded(u, clen - 1, a.topk, a.W, cidx, 0.f, ns);
    const DecodeWs ws = decode_ws(a.ws, a.B * a.H, a.units, D);
    if (p.rows > 0) {
        const int rows = p.rows;
        const T *k0 = static_cast<const T *>(a.K.ptr) + b * a.K.sb + hk * a.K.sh + (int64_t)p.start * a.K.st;
        const T *v0 = static_cast<const T *>(a.V.ptr) + b * a.V.sb + hk * a.V.sh + (int64_t)p.start * a.V.st;
        const T *q0 = static_cast<const T *>(a.Q.ptr) + b * a.Q.sb + h0 * a.Q.sh;
        for (int i = tid; i < rows * Cfg::kRowUnits; i += kThreads) {
            const int r = i / Cfg::kRowUnits, un = i % Cfg::kRowUnits;
            cp_async16(kt + i * 16, reinterpret_cast<const uint8_t *>(k0 + r * a.K.st) + un * 16);
        }
        for (int i = tid; i < GG * Cfg::kRowUnits; i += kThreads) {
            const int hh = i / Cfg::kRowUnits, un = i % Cfg::kRowUnits;
            cp_async16(qsm + i * 16, reinterpret_cast<const uint8_t *>(q0 + hh * a.Q.sh) + un * 16);
        }
        cp_async_commit();
        for (int i = tid; i < rows * Cfg::kRowUnits; i += kThreads) {
            const int r = i / Cfg::kRowUnits, un = i % Cfg::kRowUnits;
            cp_async16(vt + i * 16, reinterpret_cast<const uint8_t *>(v0 + r * a.V.st) + un * 16);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        {  // logits: a thread pair per key row, every head's dot product from one read of the row
            const int row = tid >> 1, half = tid & 1;
            const uint4 *krow = reinterpret_cast<const uint4 *>(kt + row * Cfg::kRowBytes);
            const uint4 *qv = reinterpret_cast<const uint4 *>(qsm);
            float acc[GG];
#pragma unroll
            for (int hh = 0; hh < GG; ++hh) acc[hh] = 0.f;
            if (row < rows) {
#pragma unroll
                for (int k = 0; k < Cfg::kHalfUnits; ++k) {
                    const int un = half * Cfg::kHalfUnits + rotated_unit<Cfg::kHalfUnits>(k, row, half);
                    const uint4 kv = krow[un];
#pragma unroll
                    for (int hh = 0; hh < GG; ++hh) acc[hh] = dot16<T>(kv, qv[hh * Cfg::kRowUnits + un], acc[hh]);
                }
            }
#pragma unroll
            for (int hh = 0; hh < GG; ++hh) {
                const float v = acc[hh] + __shfl_xor_sync(kFull, acc[hh], 1);
                if (half == 0) logit[hh * kChunk + row] = row < rows ? v * a.scale : -INFINITY;
            }
        }
        __syncthreads();
        for (int hh = warp; hh < GG; hh += kThreads / 32) {  // softmax: a warp per head
            const float l0 = logit[hh * kChunk + lane], l1 = logit[hh * kChunk + lane + 32];
            const float m = warp_max(fmaxf(l0, l1));
            const float e0 = expf(l0 - m), e1 = expf(l1 - m);
            const float z = warp_sum(e0 + e1);
            const float inv = 1.f / z;
            prob[hh * kChunk + lane] = e0 * inv;
            prob[hh * kChunk + lane + 32] = e1 * inv;
            if (lane == 0) lse_h[hh] = m + logf(z);
        }
        cp_async_wait<0>();
        __syncthreads();
        {  // o_u = P V for every head from one read of each V element
            const int cu = tid % Cfg::kColUnits, rg = tid / Cfg::kColUnits;
            float a0[GG], a1[GG];
#pragma unroll
            for (int hh = 0; hh < GG; ++hh) a0[hh] = a1[hh] = 0.f;
            for (int j = rg; j < rows; j += Cfg::kRowGroups) {
                const float2 vv = load2(reinterpret_cast<const T *>(vt + j * Cfg::kRowBytes) + 2 * cu);
#pragma unroll
                for (int hh = 0; hh < GG; ++hh) {
                    const float pj = prob[hh * kChunk + j];
                    a0[hh] = fmaf(pj, vv.x, a0[hh]);
                    a1[hh] = fmaf(pj, vv.y, a1[hh]);
                }
            }
#pragma unroll
            for (int hh = 0; hh < GG; ++hh) {
                red[(hh * Cfg::kRowGroups + rg) * D + 2 * cu] = a0[hh];
                red[(hh * Cfg::kRowGroups + rg) * D + 2 * cu + 1] = a1[hh];
            }
        }
        __syncthreads();
        for (int e = tid; e < GG * D; e += kThreads) {
            const int hh = e / D, x = e - hh * D;
            float v = red[hh * Cfg::kRowGroups * D + x];
#pragma unroll
            for (int g = 1; g < Cfg::kRowGroups; ++g) v += red[(hh * Cfg::kRowGroups + g) * D + x];
            ws.vec[((size_t)(qi0 + hh) * a.units + u) * D + x] = v;
        }
        if (tid < GG)
            ws.mass[(qi0 + tid) * a.units + u] = p.is_chunk ? a.score[(qi0 + tid) * a.topk + u] : lse_h[tid];
    } else {
        // an empty unit contributes weight 0 to every head
        for (int e = tid; e < GG * D; e += kThreads) {
            const int hh = e / D, x = e - hh * D;
            ws.vec[((size_t)(qi0 + hh) * a.units + u) * D + x] = 0.f;
        }
        if (tid < GG) ws.mass[(qi0 + tid) * a.units + u] = -INFINITY;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = atomicAdd(&ws.counters[qg], 1) == a.units - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    combine_group<D, GG>(ws.mass + (size_t)qi0 * a.units, ws.vec + (size_t)qi0 * a.units * D, a.units, red);
    for (int hh = 0; hh < GG; ++hh)
        store_output<T, D>(a, b, h0 + hh, 0, qi0 + hh, red + hh * (D + 1), red[hh * (D + 1) + D]);
    if (tid == 0) ws.counters[qg] = 0;
}

// General prefill path: one CTA per query, units in turn, running combination.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) attend_prefill_general_kernel(AttendArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const UnitSmem s = unit_smem<T, D>(smem);
    const int64_t qi = blockIdx.x;
    const int i = (int)(qi % a.Lq);
    const int h = (int)((qi / a.Lq) % a.H);
    const int b = (int)(qi / ((int64_t)a.Lq * a.H));
    const int t = i;
    const int hk = h / a.G;                                                 // key-value head of h
    const int64_t qg = ((int64_t)b * (a.H / a.G) + hk) * a.Lq + i;         // the group's kept list
    const int nsel = a.topk > 0 ? a.nsel[qg] : 0;
    const T *qrow = static_cast<const T *>(a.Q.ptr) + b * a.Q.sb + h * a.Q.sh + i * a.Q.st;
    const T *kh = static_cast<const T *>(a.K.ptr) + b * a.K.sb + hk * a.K.sh;
    const T *vh = static_cast<const T *>(a.V.ptr) + b * a.V.sb + hk * a.V.sh;
    // thread x (< D) owns output column x
    float M = -INFINITY, zsum = 0.f, acc = 0.f;
    for (int u = 0; u < a.units; ++u) {
        const UnitPlan p = plan_unit(u, t, a.topk, a.W, a.idx + qg * a.topk, a.score + qi * a.topk, nsel);
        if (p.rows == 0) continue;
        unit_issue<T, D>(s, qrow, kh + (int64_t)p.start * a.K.st, a.K.st, vh + (int64_t)p.start * a.V.st,
                         a.V.st, p.rows);
        const float lse_tile = unit_compute<T, D>(s, p.rows, a.scale);
        const float m = p.is_chunk ? p.mass : lse_tile;
        if (m != -INFINITY) {
            const float Mn = fmaxf(M, m);
            const float fo = expf(M - Mn), fn = expf(m - Mn);
            zsum = zsum * fo + fn;
            if (threadIdx.x < D) acc = acc * fo + fn * s.red[threadIdx.x];
            M = Mn;
        }
        __syncthreads();  // shared tiles are rewritten by the next unit
    }
    float *o = s.red;
    if (threadIdx.x < D) o[threadIdx.x] = M == -INFINITY ? 0.f : acc / zsum;
    __syncthreads();
    store_output<T, D>(a, b, h, i, qi, o, M == -INFINITY ? -INFINITY : M + logf(zsum));
}

template <typename T, int D, int GG>
hils_status launch_decode_group(const AttendArgs &a, cudaStream_t st) {
    using Cfg = GroupUnitCfg<T, D, GG>;
    static KernelSetup setup;
    const hils_status stt = kernel_setup(setup, (const void *)attend_decode_group_kernel<T, D, GG>, kThreads,
                                         Cfg::kSmemBytes, nullptr);
    if (stt != HILS_OK) return stt;
    return launch_dependent((const void *)attend_decode_group_kernel<T, D, GG>, dim3(a.units, a.B * (a.H / GG)),
                            dim3(kThreads), Cfg::kSmemBytes, st, a);
}

template <typename T, int D>
hils_status launch_decode(const AttendArgs &a, cudaStream_t st) {
    using Cfg = UnitCfg<T, D>;
    const int nq = a.B * a.H;
    if (nq == 0) return HILS_OK;
    // groups of 2, 4 or 8 heads share each unit's copies; other group sizes take a CTA
    // per head
    if (a.G == 2) return launch_decode_group<T, D, 2>(a, st);
    if (a.G == 4) return launch_decode_group<T, D, 4>(a, st);
    if (a.G == 8) return launch_decode_group<T, D, 8>(a, st);
    static KernelSetup setup;
    const hils_status stt = kernel_setup(setup, (const void *)attend_decode_kernel<T, D>, kThreads,
                                         Cfg::kSmemBytes, nullptr);
    if (stt != HILS_OK) return stt;
    return launch_dependent((const void *)attend_decode_kernel<T, D>, dim3(a.units, nq), dim3(kThreads),
                            Cfg::kSmemBytes, st, a);
}

template <typename T, int D>
hils_status launch_prefill_general(const AttendArgs &a, cudaStream_t st) {
    using Cfg = UnitCfg<T, D>;
    const int64_t nq = (int64_t)a.B * a.H * a.Lq;
    if (nq == 0) return HILS_OK;
    static KernelSetup setup;
    const hils_status stt = kernel_setup(setup, (const void *)attend_prefill_general_kernel<T, D>, kThreads,
                                         Cfg::kSmemBytes, nullptr);
    if (stt != HILS_OK) return stt;
    attend_prefill_general_kernel<T, D><<<(unsigned)nq, kThreads, Cfg::kSmemBytes, st>>>(a);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace

size_t attend_decode_ws_bytes(int queries, int units, int d) {
    return attend_decode_counter_bytes(queries) + align256((size_t)queries * units * sizeof(float)) +
           (size_t)queries * units * d * sizeof(float);
}

hils_status launch_attend_decode(hils_dtype dt, int d, const AttendArgs &a, cudaStream_t s) {
    if (dt == HILS_BF16) return d == 64 ? launch_decode<bf16, 64>(a, s) : launch_decode<bf16, 128>(a, s);
    return d == 64 ? launch_decode<float, 64>(a, s) : launch_decode<float, 128>(a, s);
}

hils_status launch_attend_prefill_general(hils_dtype dt, int d, const AttendArgs &a, cudaStream_t s) {
    if (dt == HILS_BF16)
        return d == 64 ? launch_prefill_general<bf16, 64>(a, s) : launch_prefill_general<bf16, 128>(a, s);
    return d == 64 ? launch_prefill_general<float, 64>(a, s) : launch_prefill_general<float, 128>(a, s);
}

}  // namespace hils
