// Backward pass of the HiLS-Attention forward for a fixed selection: "Hierarchical
// Sparse Attention Done Right" (picx.dev summary), Methodology 1-2, Eq. 7, Eq. 8 and
// Eq. 10, differentiated by hand. Top-K is piecewise constant, so the gradient of the
// output o_i reaches the inputs through the kept chunks' scores s^_{i,c}, the token
// logits l_ij = scale q_i . k_j and the values, and from the scores through the summaries
// (k'_c, b'_c) into the keys and the landmark queries.
//
// With w_u = exp(m_u - lse_i) the weight of unit u in Eq. 10 (m_u = s^_{i,c} for a kept
// chunk, l_ij for a window token) and D_i = dO_i . o_i:
//   kept chunk c:  p_j = softmax over the chunk of l_ij, o_c = sum_j p_j v_j,
//                  ds^_{i,c} = w_c (dO_i . o_c - D_i),
//                  dl_ij = w_c p_j (dO_i . v_j - dO_i . o_c),  dv_j += w_c p_j dO_i;
//   window token j: dl_ij = w_j (dO_i . v_j - D_i),  dv_j += w_j dO_i;
//   dq_i = scale sum_j dl_ij k_j,  dk_j += scale dl_ij q_i.
// Eq. 7: dq~_i = scale sum_c ds^_{i,c} k'_c,  dk'_c += scale ds^_{i,c} q~_i,
//        db'_c += ds^_{i,c}.
// Eq. 8 with p = softmax(scale q'_c . k_j) over the chunk:
//   dp_j = k_j . dk'_c - db'_c (log p_j + 1),  dl_j = p_j (dp_j - sum_i p_i dp_i),
//   dq'_c = scale sum_j dl_j k_j,  dk_j += p_j dk'_c + scale dl_j q'_c.
//
// One 128-thread CTA per query (attend, score) or per chunk (summaries); the key and
// value gradients, which many queries and chunks share, are accumulated with float32
// atomic adds (the order of the additions is not fixed). Gradients are float32, dense.
#include <math.h>

#include "hils_internal.cuh"

namespace hils {
namespace {

constexpr int kThreads = 128;

template <typename T, int D>
struct BwdCfg {
    // key and value rows of one unit as float32, then the per-row scalars
    static constexpr int kSmemBytes = (2 * kChunk * D + 3 * D + 6 * kChunk + 8) * 4;
};

template <typename T>
__device__ __forceinline__ float elem(const T *p, int x) {
    if constexpr (sizeof(T) == 2) return __bfloat162float(p[x]);
    else return p[x];
}

__device__ __forceinline__ float block_sum(float v, float *scratch) {
    v = warp_sum(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) r += scratch[w];
    return r;
}

// grid: B*H*N, one query each.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) attend_backward_kernel(BwdAttendArgs a) {
    extern __shared__ __align__(16) float fsm[];
    float *kt = fsm, *vt = kt + kChunk * D;          // [64][D] each
    float *qf = vt + kChunk * D, *dof = qf + D, *of = dof + D;
    float *lg = of + D, *tj = lg + kChunk, *dl = tj + kChunk, *cv = dl + kChunk;
    float *scratch = cv + kChunk;                     // 8 floats
    const int tid = threadIdx.x;
    const int64_t qi = blockIdx.x;
    const int i = (int)(qi % a.N);
    const int h = (int)((qi / a.N) % a.H);
    const int b = (int)(qi / ((int64_t)a.N * a.H));
    const int Hk = a.H / a.G, hk = h / a.G;
    const int64_t qg = ((int64_t)b * Hk + hk) * a.N + i;
    const T *qrow = static_cast<const T *>(a.Q.ptr) + b * a.Q.sb + h * a.Q.sh + (int64_t)i * a.Q.st;
    const T *orow = static_cast<const T *>(a.O.ptr) + b * a.O.sb + h * a.O.sh + (int64_t)i * a.O.st;
    const float *dorow = a.dO + qi * D;
    for (int x = tid; x < D; x += kThreads) {
        qf[x] = elem(qrow, x);
        dof[x] = dorow[x];
        of[x] = elem(orow, x);
    }
    __syncthreads();
    float part = 0.f;
    for (int x = tid; x < D; x += kThreads) part = fmaf(dof[x], of[x], part);
    const float Di = block_sum(part, scratch);  // dO . o
    const float lse = a.lse[qi];
    const int K = a.topk;
    const int ns = (K > 0 && isfinite(lse)) ? min(max(a.nsel[qg], 0), K) : 0;
    float dq = 0.f;  // column tid of dq (tid < D)
    const int w0 = max(0, i - a.W + 1);
    const int nwin = (a.W > 0 && isfinite(lse)) ? (i - w0) / kChunk + 1 : 0;
    const T *kbase = static_cast<const T *>(a.K.ptr) + b * a.K.sb + hk * a.K.sh;
    const T *vbase = static_cast<const T *>(a.V.ptr) + b * a.V.sb + hk * a.V.sh;
    float *dkbase = a.dK + ((int64_t)b * Hk + hk) * a.N * D;
    float *dvbase = a.dV + ((int64_t)b * Hk + hk) * a.N * D;
    for (int u = 0; u < ns + nwin; ++u) {
        const bool chunk = u < ns;
        int start, rows;
        float mass = 0.f;
        if (chunk) {
            const int c = a.idx[qg * K + u];
            start = c * kChunk;
            rows = kChunk;
            mass = a.score[qi * K + u];
        } else {
            start = w0 + (u - ns) * kChunk;
            rows = min(kChunk, i - start + 1);
        }
        for (int e = tid; e < rows * D; e += kThreads) {
            const int j = e / D, x = e - (e / D) * D;
            kt[e] = elem(kbase + (int64_t)(start + j) * a.K.st, x);
            vt[e] = elem(vbase + (int64_t)(start + j) * a.V.st, x);
        }
        __syncthreads();
        {  // l_j = scale q . k_j and t_j = dO . v_j, two threads per row
            const int row = tid >> 1, half = tid & 1;
            float al = 0.f, at = 0.f;
            if (row < rows) {
                for (int x = half * (D / 2); x < (half + 1) * (D / 2); ++x) {
                    al = fmaf(qf[x], kt[row * D + x], al);
                    at = fmaf(dof[x], vt[row * D + x], at);
                }
            }
            al += __shfl_xor_sync(kFull, al, 1);
            at += __shfl_xor_sync(kFull, at, 1);
            if (half == 0 && row < kChunk) {
                lg[row] = row < rows ? al * a.scale : -INFINITY;
                tj[row] = row < rows ? at : 0.f;
            }
        }
        __syncthreads();
        if (tid < 32) {
            const int lane = tid;
            const float l0 = lg[lane], l1 = lg[lane + 32];
            if (chunk) {
                const float m = warp_max(fmaxf(l0, l1));
                const float e0 = expf(l0 - m), e1 = expf(l1 - m);
                const float inv = 1.f / warp_sum(e0 + e1);
                const float p0 = e0 * inv, p1 = e1 * inv;
                const float oc = warp_sum(p0 * tj[lane] + p1 * tj[lane + 32]);  // dO . o_c
                const float w = expf(mass - lse);
                dl[lane] = w * p0 * (tj[lane] - oc);
                dl[lane + 32] = w * p1 * (tj[lane + 32] - oc);
                cv[lane] = w * p0;
                cv[lane + 32] = w * p1;
                if (lane == 0) a.dscore[qi * K + u] = w * (oc - Di);
            } else {
                const float w0j = expf(l0 - lse), w1j = expf(l1 - lse);  // 0 past the rows
                dl[lane] = w0j * (tj[lane] - Di);
                dl[lane + 32] = w1j * (tj[lane + 32] - Di);
                cv[lane] = w0j;
                cv[lane + 32] = w1j;
            }
        }
        __syncthreads();
        if (tid < D) {
            float acc = 0.f;
            for (int j = 0; j < rows; ++j) acc = fmaf(dl[j], kt[j * D + tid], acc);
            dq = fmaf(a.scale, acc, dq);
        }
        for (int e = tid; e < rows * D; e += kThreads) {
            const int j = e / D, x = e - (e / D) * D;
            atomicAdd(dkbase + (int64_t)(start + j) * D + x, a.scale * dl[j] * qf[x]);
            atomicAdd(dvbase + (int64_t)(start + j) * D + x, cv[j] * dof[x]);
        }
        __syncthreads();  // the unit's rows are no longer read
    }
    if (tid < D) a.dQ[qi * D + tid] = dq;
    for (int k = ns + tid; k < K; k += kThreads) a.dscore[qi * K + k] = 0.f;
}

// grid: B*H*Lq, one query each: Eq. 7 backward.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) select_backward_kernel(BwdSelectArgs a) {
    const int tid = threadIdx.x;
    const int64_t qi = blockIdx.x;
    const int i = (int)(qi % a.Lq);
    const int h = (int)((qi / a.Lq) % a.H);
    const int b = (int)(qi / ((int64_t)a.Lq * a.H));
    const int Hk = a.H / a.G;
    const int64_t qg = ((int64_t)b * Hk + h / a.G) * a.Lq + i;
    const int K = a.topk;
    const int ns = K > 0 ? min(max(a.nsel[qg], 0), K) : 0;
    const T *qrow = static_cast<const T *>(a.Qcal.ptr) + b * a.Qcal.sb + h * a.Qcal.sh + (int64_t)i * a.Qcal.st;
    const T *khead = static_cast<const T *>(a.Ksum.ptr) + b * a.Ksum.sb + h * a.Ksum.sh;
    float *dks = a.dKsum + ((int64_t)b * a.H + h) * a.C * D;
    float *dbs = a.dBsum + ((int64_t)b * a.H + h) * a.C;
    if (tid >= D) return;
    const float qx = elem(qrow, tid);
    float acc = 0.f;
    for (int k = 0; k < ns; ++k) {
        const int c = a.idx[qg * K + k];
        const float ds = a.dscore[qi * K + k];
        acc = fmaf(ds, elem(khead + (int64_t)c * a.Ksum.st, tid), acc);
        atomicAdd(dks + (int64_t)c * D + tid, a.scale * ds * qx);
        if (tid == 0) atomicAdd(dbs + c, ds);
    }
    a.dQcal[qi * D + tid] = a.scale * acc;
}

// grid: B*H*C, one chunk each: Eq. 8 backward.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) summarize_backward_kernel(BwdSummarizeArgs a) {
    extern __shared__ __align__(16) float fsm[];
    float *kt = fsm;                                  // [64][D]
    float *qf = kt + kChunk * D, *dk = qf + D;
    float *pr = dk + D, *dl = pr + kChunk;
    float *scratch = dl + kChunk;
    const int tid = threadIdx.x;
    const int64_t u = blockIdx.x;
    const int c = (int)(u % a.C);
    const int h = (int)((u / a.C) % a.H);
    const int b = (int)(u / ((int64_t)a.C * a.H));
    const int Hk = a.H / a.G, hk = h / a.G;
    const T *kbase = static_cast<const T *>(a.K.ptr) + b * a.K.sb + hk * a.K.sh + (int64_t)c * kChunk * a.K.st;
    const T *lq = static_cast<const T *>(a.LQ.ptr) + b * a.LQ.sb + h * a.LQ.sh + (int64_t)c * a.LQ.st;
    const float db = a.dBsum[u];
    for (int e = tid; e < kChunk * D; e += kThreads) {
        const int j = e / D, x = e - (e / D) * D;
        kt[e] = elem(kbase + (int64_t)j * a.K.st, x);
    }
    for (int x = tid; x < D; x += kThreads) {
        qf[x] = elem(lq, x);
        dk[x] = a.dKsum[u * D + x];
    }
    __syncthreads();
    float lj = -INFINITY, kd = 0.f;  // row tid / 2: logit and k_j . dk'
    {
        const int row = tid >> 1, half = tid & 1;
        float al = 0.f, ak = 0.f;
        for (int x = half * (D / 2); x < (half + 1) * (D / 2); ++x) {
            al = fmaf(qf[x], kt[row * D + x], al);
            ak = fmaf(dk[x], kt[row * D + x], ak);
        }
        al += __shfl_xor_sync(kFull, al, 1);
        ak += __shfl_xor_sync(kFull, ak, 1);
        lj = al * a.scale;
        kd = ak;
    }
    // softmax over the 64 rows (each row held by a thread pair: halve the sums)
    const float m = [&] {
        float v = warp_max(lj);
        __syncthreads();
        if ((tid & 31) == 0) scratch[tid >> 5] = v;
        __syncthreads();
        float r = scratch[0];
        for (int w = 1; w < kThreads / 32; ++w) r = fmaxf(r, scratch[w]);
        return r;
    }();
    const float ej = expf(lj - m);
    const float z = 0.5f * block_sum(ej, scratch);
    const float pj = ej / z;
    const float logp = (lj - m) - logf(z);
    const float dp = kd - db * (logp + 1.f);
    const float spd = 0.5f * block_sum(pj * dp, scratch);
    const float dlj = pj * (dp - spd);
    if ((tid & 1) == 0) {
        pr[tid >> 1] = pj;
        dl[tid >> 1] = dlj;
    }
    __syncthreads();
    float *dkbase = a.dK + ((int64_t)b * Hk + hk) * a.N * D + (int64_t)c * kChunk * D;
    if (tid < D) {
        float acc = 0.f;
        for (int j = 0; j < kChunk; ++j) acc = fmaf(dl[j], kt[j * D + tid], acc);
        a.dLQ[u * D + tid] = a.scale * acc;
    }
    for (int e = tid; e < kChunk * D; e += kThreads) {
        const int j = e / D, x = e - (e / D) * D;
        atomicAdd(dkbase + (int64_t)j * D + x, fmaf(pr[j], dk[x], a.scale * dl[j] * qf[x]));
    }
}

template <typename T, int D>
hils_status launch_attend_bwd(const BwdAttendArgs &a, cudaStream_t s) {
    constexpr int smem = BwdCfg<T, D>::kSmemBytes;
    static KernelSetup setup;
    const hils_status st = kernel_setup(setup, (const void *)attend_backward_kernel<T, D>, kThreads, smem, nullptr);
    if (st != HILS_OK) return st;
    attend_backward_kernel<T, D><<<(unsigned)((int64_t)a.B * a.H * a.N), kThreads, smem, s>>>(a);
    return record_cuda_error(cudaGetLastError());
}

template <typename T, int D>
hils_status launch_select_bwd(const BwdSelectArgs &a, cudaStream_t s) {
    select_backward_kernel<T, D><<<(unsigned)((int64_t)a.B * a.H * a.Lq), kThreads, 0, s>>>(a);
    return record_cuda_error(cudaGetLastError());
}

template <typename T, int D>
hils_status launch_summarize_bwd(const BwdSummarizeArgs &a, cudaStream_t s) {
    constexpr int smem = (kChunk * D + 2 * D + 2 * kChunk + 8) * 4;
    static KernelSetup setup;
    const hils_status st = kernel_setup(setup, (const void *)summarize_backward_kernel<T, D>, kThreads, smem, nullptr);
    if (st != HILS_OK) return st;
    summarize_backward_kernel<T, D><<<(unsigned)((int64_t)a.B * a.H * a.C), kThreads, smem, s>>>(a);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace

hils_status launch_attend_backward(hils_dtype dt, int d, const BwdAttendArgs &a, cudaStream_t s) {
    if ((int64_t)a.B * a.H * a.N == 0) return HILS_OK;
    if (dt == HILS_BF16) return d == 64 ? launch_attend_bwd<bf16, 64>(a, s) : launch_attend_bwd<bf16, 128>(a, s);
    return d == 64 ? launch_attend_bwd<float, 64>(a, s) : launch_attend_bwd<float, 128>(a, s);
}

hils_status launch_select_backward(hils_dtype dt, int d, const BwdSelectArgs &a, cudaStream_t s) {
    if ((int64_t)a.B * a.H * a.Lq == 0) return HILS_OK;
    if (dt == HILS_BF16) return d == 64 ? launch_select_bwd<bf16, 64>(a, s) : launch_select_bwd<bf16, 128>(a, s);
    return d == 64 ? launch_select_bwd<float, 64>(a, s) : launch_select_bwd<float, 128>(a, s);
}

hils_status launch_summarize_backward(hils_dtype dt, int d, const BwdSummarizeArgs &a, cudaStream_t s) {
    if ((int64_t)a.B * a.H * a.C == 0) return HILS_OK;
    if (dt == HILS_BF16)
        return d == 64 ? launch_summarize_bwd<bf16, 64>(a, s) : launch_summarize_bwd<bf16, 128>(a, s);
    return d == 64 ? launch_summarize_bwd<float, 64>(a, s) : launch_summarize_bwd<float, 128>(a, s);
}

}  // namespace hils
