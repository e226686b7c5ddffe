// One pipeline stage of the chunk screen (Eq. 7 of "Hierarchical Sparse Attention Done
// Right" (picx.dev summary), with the rigorous radius of the exact selection): the
// stage layout, the cooperative copies that fill it, and the screen of its rows on CUDA
// cores, for the decode select's screen kernel.
#pragma once
#include "select_pick.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

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

// Screen of one stage on CUDA cores (all threads), float32 arithmetic for either input
// type: kTPR threads share a row (one 16-byte unit each), each accumulates its unit's
// partial dot and |k|^2 for kRPT rows with packed float32 FMAs, and a transpose
// reduction across the kTPR lanes leaves each lane the totals of one row. Radius: any
// order of the float32 sums stays within (d+1) 2^-24 sum|q k| <= (d+1) 2^-24 |q~| |k'|
// (Cauchy-Schwarz), doubled, plus 2^-22 |s| for the final fused multiply-add:
//   e_c = scale |q~| |k'_c| (d+2) 2^-23 + |s_c| 2^-22.
// bf16 rows sit as TMA wrote them with the 128-byte swizzle (16-byte unit u of row r in
// column block u / 8 at r * 128 + ((u % 8) ^ (r % 8)) * 16), float32 rows plainly.
template <typename T, int D, typename Cfg>
__device__ void screen_stage_fma(const uint8_t *st, float scale, int c0, int ne, float2 *out, int base,
                                 float2 *gscr) {
    constexpr int kN = Vec<T>::kN;
    const int tid = threadIdx.x, col = tid % Cfg::kTPR, rg = tid / Cfg::kTPR;
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
        const int row = rg * Cfg::kRPT + r;
        const uint8_t *unit = Cfg::kTma ? st + (col >> 3) * (Cfg::kRows * 128) + row * 128 + (((col & 7) ^ (row & 7)) << 4)
                                        : st + row * Cfg::kRowBytes + col * 16;
        const uint4 kv = *reinterpret_cast<const uint4 *>(unit);
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
    const float ecoef = scale * sqrtf(qn2) * ((float)(D + 2) * 0x1p-23f);
    const float sv = fmaf(dotv[0], scale, reinterpret_cast<const float *>(st + Cfg::kBiasOff)[row]);
    const float ev = fmaf(ecoef, sqrt_approx(ksqv[0]), fabsf(sv) * 0x1p-22f);
    if (valid && (col & 1) == 0) out[c - base] = make_float2(sv, ev);
    float gs = valid ? sv : -INFINITY, ge = valid ? ev : 0.f;
#pragma unroll
    for (int o = Cfg::kTPR / 2; o > 0; o >>= 1) {
        gs = fmaxf(gs, __shfl_xor_sync(kFull, gs, o));
        ge = fmaxf(ge, __shfl_xor_sync(kFull, ge, o));
    }
    if (col == 0) gscr[rg] = make_float2(gs, ge);
}

// Layout of one pipeline stage of ROWS summary rows screened by NT threads: the rows
// (bf16: 128-byte column blocks written by TMA with the 128-byte swizzle, see
// screen_stage_fma; float32: plain rows), their biases, the query row and the query's
// position. bf16 stages start on 1024-byte boundaries (the swizzle's period).
template <typename T, int D, int NT, int ROWS>
struct StageCfg {
    static constexpr int kThreads = NT;
    static constexpr int kRows = ROWS;
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kTPR = kRowBytes / 16;     // threads per row: 8, 16 or 32
    static constexpr int kRowGroups = NT / kTPR;    // rows per step
    static constexpr int kRPT = ROWS / kRowGroups;  // rows per thread
    static constexpr int kBiasOff = ROWS * kRowBytes;
    static constexpr int kQOff = kBiasOff + ROWS * 4;
    static constexpr int kPosOff = kQOff + kRowBytes;
    static constexpr int kStageBytes = sizeof(T) == 2 ? (kPosOff + 16 + 1023) / 1024 * 1024 : kPosOff + 16;
    static constexpr int kGroupsPerBlock = ROWS / kGroupRows;
    static constexpr int kCopies = ROWS * kTPR / NT;  // 16-byte copies per thread
    static_assert(2 * kRPT == kTPR, "half-square transpose reduction");
    // bf16 rows come by TMA (swizzled), float32 rows by cp.async; both are screened on
    // CUDA cores, kRPT rows per group of kTPR threads
    static constexpr bool kTma = sizeof(T) == 2;
    static constexpr int kSlotRows = kRPT;
    static constexpr int kSlots = ROWS / kSlotRows;
    static constexpr int kSlotsPerGroup = kGroupRows / kSlotRows;
};

// Every thread issues its share of the cp.async copies of one stage: `rows` summary
// rows from `kh` (row stride kst elements) starting at chunk c0 (float32 only: bf16 rows
// come by TMA), their biases, the query row, and the position (from `pos` if not null,
// else the value `pos_value`).
template <typename T, typename Cfg>
__device__ __forceinline__ void stage_issue(uint8_t *st, const T *kh, int64_t kst, int c0, int rows, const float *brow,
                                            const T *qrow, const int32_t *pos, int pos_value) {
    const int tid = threadIdx.x, col = tid % Cfg::kTPR;
    const int r0 = tid / Cfg::kTPR;
    if constexpr (!Cfg::kTma) {
        const uint8_t *src = reinterpret_cast<const uint8_t *>(kh + (int64_t)(c0 + r0) * kst) + col * 16;
        uint8_t *dst = st + r0 * Cfg::kRowBytes + col * 16;
        constexpr int kStep = Cfg::kThreads / Cfg::kTPR;
        const int64_t src_step = (int64_t)kStep * kst * (int64_t)sizeof(T);
#pragma unroll
        for (int k = 0; k < Cfg::kCopies; ++k)
            if (r0 + k * kStep < rows) cp_async16(dst + k * kStep * Cfg::kRowBytes, src + k * src_step);
    }
    for (int r = tid; r < rows; r += Cfg::kThreads) cp_async4(st + Cfg::kBiasOff + r * 4, brow + r);
    for (int u = tid; u < Cfg::kTPR; u += Cfg::kThreads)
        cp_async16(st + Cfg::kQOff + u * 16, reinterpret_cast<const uint8_t *>(qrow) + u * 16);
    if (tid == 0) {
        if (pos) cp_async4(st + Cfg::kPosOff, pos);
        else *reinterpret_cast<int *>(st + Cfg::kPosOff) = pos_value;
    }
}

}  // namespace
}  // namespace hils
