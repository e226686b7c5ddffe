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
// Attend: key-major. A 128-thread CTA owns one 64-key block of one (b, h) and walks the
// queries that attend it, accumulating the block's dk and dv in shared memory and adding
// each query's dq share to dQ with float32 atomics: for a window block, the contiguous
// range of queries whose window reaches it; for a chunk, the queries that kept it, from
// an inverted index of the selection built first (count, scan, scatter). D_i = dO_i . o_i
// is computed once per query beforehand. Score backward: a CTA per 256 queries of one
// head (dQcal, then its kept entries sorted by chunk and summed per chunk). Summaries: a
// CTA per chunk. Shared gradients (dK, dV, dKsum, dBsum, dQ) are float32 atomic adds, in
// no fixed order. Gradients are float32, dense. bf16 with d = 128 takes the tensor-core
// form of the walk (backward_tc.cu: 128 queries per step on tcgen05, chunk lists cut into
// runs of at most 1024 queries, one persistent CTA per SM); bf16 with d = 64 the mma.sync
// form below; float32 the CUDA-core form.
#include <math.h>

#include "backward_common.cuh"

namespace hils {
namespace {

constexpr int kThreads = 128;

// Workspace of the attend backward: a status word (256 bytes), D_i per query, then per
// (b, group) the chunk counts, starts (C + 1), cursors and the inverted index (N * K
// entries). The tensor-core walk (bf16, d = 128) adds: one record per (query head,
// index entry), the chunk items per (b, group) and their count, and contiguous bf16
// copies of dO and Q ([B*H*N][d] rows, the row gathers' source).
struct BwdWs {
    uint32_t *status;
    float *D;
    int *count, *start, *cursor, *entries;
    int4 *recs, *items;
    int *nitems;
    bf16 *dOb, *Qc;
    int max_items;
    size_t bytes;
};
inline size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }
inline bool bwd_tc_layout(hils_dtype dt, int d) { return dt == HILS_BF16 && d == 128; }
inline BwdWs bwd_ws(void *ws, bool tc, int B, int H, int Hk, int N, int K, int d) {
    const int C = N / kChunk;
    uint8_t *p = static_cast<uint8_t *>(ws);
    BwdWs w = {};
    size_t off = 0;
    w.status = reinterpret_cast<uint32_t *>(p + off);
    off += 256;
    w.D = reinterpret_cast<float *>(p + off);
    off += a256((size_t)B * H * N * 4);
    w.count = reinterpret_cast<int *>(p + off);
    off += a256((size_t)B * Hk * C * 4);
    w.start = reinterpret_cast<int *>(p + off);
    off += a256((size_t)B * Hk * (C + 1) * 4);
    w.cursor = reinterpret_cast<int *>(p + off);
    off += a256((size_t)B * Hk * C * 4);
    w.entries = reinterpret_cast<int *>(p + off);
    off += a256((size_t)B * Hk * N * (K > 0 ? K : 1) * 4);
    if (tc) {
        // chunk items: sum over chunks of ceil(count / kBwdItemQueries) <= C + N K / kBwdItemQueries
        w.max_items = C + (int)(((int64_t)N * K + kBwdItemQueries - 1) / kBwdItemQueries);
        w.recs = reinterpret_cast<int4 *>(p + off);
        off += a256((size_t)B * H * N * K * 16);
        w.items = reinterpret_cast<int4 *>(p + off);
        off += a256((size_t)B * Hk * w.max_items * 16);
        w.nitems = reinterpret_cast<int *>(p + off);
        off += a256((size_t)B * Hk * 4);
        w.dOb = reinterpret_cast<bf16 *>(p + off);
        off += a256((size_t)B * H * N * d * 2);
        w.Qc = reinterpret_cast<bf16 *>(p + off);
        off += a256((size_t)B * H * N * d * 2);
    }
    w.bytes = off;
    return w;
}

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

// ---- key-major attend backward

// D_i = dO_i . o_i, one warp per query.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) bwd_dot_kernel(BwdAttendArgs a, float *Dv) {
    const int64_t qi = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (qi >= (int64_t)a.B * a.H * a.N) return;
    const int i = (int)(qi % a.N);
    const int h = (int)((qi / a.N) % a.H);
    const int b = (int)(qi / ((int64_t)a.N * a.H));
    const T *orow = static_cast<const T *>(a.O.ptr) + b * a.O.sb + h * a.O.sh + (int64_t)i * a.O.st;
    float acc = 0.f;
    for (int x = lane; x < D; x += 32) acc = fmaf(a.dO[qi * D + x], elem(orow, x), acc);
    acc = warp_sum(acc);
    if (lane == 0) Dv[qi] = acc;
}

// The tensor-core walk's preparation (bf16, d = 128), one warp per query row: D_i, and
// the row of dO rounded to bf16 and the row of Q, both into contiguous [B*H*N][128]
// arrays (lane l holds elements 4l..4l+3).
__global__ void __launch_bounds__(kThreads) bwd_prep_kernel(BwdAttendArgs a, float *Dv, bf16 *dOb, bf16 *Qc) {
    const int64_t qi = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (qi >= (int64_t)a.B * a.H * a.N) return;
    const int i = (int)(qi % a.N);
    const int h = (int)((qi / a.N) % a.H);
    const int b = (int)(qi / ((int64_t)a.N * a.H));
    const bf16 *orow = static_cast<const bf16 *>(a.O.ptr) + b * a.O.sb + h * a.O.sh + (int64_t)i * a.O.st;
    const bf16 *qrow = static_cast<const bf16 *>(a.Q.ptr) + b * a.Q.sb + h * a.Q.sh + (int64_t)i * a.Q.st;
    const float *g = a.dO + qi * 128 + 4 * lane;
    const float g0 = g[0], g1 = g[1], g2 = g[2], g3 = g[3];
    const uint2 ov = *reinterpret_cast<const uint2 *>(orow + 4 * lane);
    const uint2 qv = *reinterpret_cast<const uint2 *>(qrow + 4 * lane);
    float acc = g0 * bf16lo(ov.x);
    acc = fmaf(g1, bf16hi(ov.x), acc);
    acc = fmaf(g2, bf16lo(ov.y), acc);
    acc = fmaf(g3, bf16hi(ov.y), acc);
    acc = warp_sum(acc);
    if (lane == 0) Dv[qi] = acc;
    const __nv_bfloat162 d01 = __floats2bfloat162_rn(g0, g1), d23 = __floats2bfloat162_rn(g2, g3);
    *reinterpret_cast<uint2 *>(dOb + qi * 128 + 4 * lane) =
        make_uint2(*reinterpret_cast<const uint32_t *>(&d01), *reinterpret_cast<const uint32_t *>(&d23));
    *reinterpret_cast<uint2 *>(Qc + qi * 128 + 4 * lane) = qv;
}

// Inverted index of the selection per (b, group): count[c], then (after the scan)
// cursor[c] = start[c] + filled so far; entries hold i * 32 + k.
__global__ void bwd_count_kernel(BwdAttendArgs a, int *count) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // (b, group, i, k)
    const int Hk = a.H / a.G, K = a.topk;
    if (e >= (int64_t)a.B * Hk * a.N * K) return;
    const int64_t qg = e / K;
    const int k = (int)(e % K);
    if (k >= min(max(a.nsel[qg], 0), K)) return;
    const int c = a.idx[e];
    const int64_t bg = qg / a.N;
    if (c >= 0 && c < a.N / kChunk) atomicAdd(&count[bg * (a.N / kChunk) + c], 1);
}

// exclusive scan of count over the C chunks of one (b, group): start[c], cursor[c]; with
// `items`, also the group's chunk items: chunk c's entries cut into runs of at most
// kBwdItemQueries, {c, first entry, end entry, 0}, in chunk order, and their number.
__global__ void __launch_bounds__(1024) bwd_scan_kernel(int C, const int *count, int *start, int *cursor,
                                                        int4 *items, int *nitems, int max_items) {
    __shared__ int part[1024];
    const int64_t bg = blockIdx.x;
    const int *cnt = count + bg * C;
    const int per = (C + 1023) / 1024, t = threadIdx.x;
    const int c_lo = min(C, t * per), c_hi = min(C, (t + 1) * per);
    // inclusive scan of one value per thread, in place in part[]
    auto block_scan = [&](int v) {
        part[t] = v;
        __syncthreads();
        for (int o = 1; o < 1024; o <<= 1) {
            const int u = t >= o ? part[t - o] : 0;
            __syncthreads();
            part[t] += u;
            __syncthreads();
        }
    };
    int sum = 0;
    for (int c = c_lo; c < c_hi; ++c) sum += cnt[c];
    block_scan(sum);
    int run = part[t] - sum;
    for (int c = c_lo; c < c_hi; ++c) {
        start[bg * (C + 1) + c] = run;
        cursor[bg * C + c] = run;
        run += cnt[c];
    }
    if (t == 1023) start[bg * (C + 1) + C] = part[1023];
    if (!items) return;
    int segs = 0;
    for (int c = c_lo; c < c_hi; ++c) segs += (cnt[c] + kBwdItemQueries - 1) / kBwdItemQueries;
    run = part[t] - sum;  // this thread's first entry
    __syncthreads();
    block_scan(segs);
    int o = part[t] - segs;
    int4 *it = items + bg * max_items;
    for (int c = c_lo; c < c_hi; ++c) {
        const int n = cnt[c];
        for (int e = 0; e < n; e += kBwdItemQueries) it[o++] = make_int4(c, run + e, run + min(n, e + kBwdItemQueries), 0);
        run += n;
    }
    if (t == 1023) nitems[bg] = part[1023];
}

// The record of index entry `pos` (query i, slot k) for each query head of group g:
// {i * 32 + k (or -1 when the row's lse is not finite), w = exp(s^_{i,c} - lse_i), D_i, i}.
__device__ __forceinline__ void write_records(const BwdAttendArgs &a, const float *Dv, int4 *recs, int b, int g,
                                              int i, int k, int pos) {
    const int K = a.topk;
    for (int hh = 0; hh < a.G; ++hh) {
        const int64_t bh = (int64_t)b * a.H + g * a.G + hh;
        const int64_t qh = bh * a.N + i;
        const float lse = a.lse[qh];
        const bool fin = isfinite(lse);
        const float w = fin ? expf(a.score[qh * K + k] - lse) : 0.f;
        recs[bh * a.N * K + pos] = make_int4(fin ? i * 32 + k : -1, __float_as_int(w), __float_as_int(Dv[qh]), i);
    }
}

// Fills the inverted index (`entries`: i * 32 + k, or null) and/or each query head's
// records of its entries (`recs`, or null); one thread per (b, group, i, k).
__global__ void bwd_scatter_kernel(BwdAttendArgs a, int *cursor, int *entries, const float *Dv, int4 *recs) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int Hk = a.H / a.G, K = a.topk, C = a.N / kChunk;
    if (e >= (int64_t)a.B * Hk * a.N * K) return;
    const int64_t qg = e / K;
    const int k = (int)(e % K);
    if (k >= min(max(a.nsel[qg], 0), K)) return;
    const int c = a.idx[e];
    if (c < 0 || c >= C) return;
    const int64_t bg = qg / a.N;
    const int i = (int)(qg % a.N);
    const int pos = atomicAdd(&cursor[bg * C + c], 1);
    if (entries) entries[bg * (int64_t)a.N * K + pos] = i * 32 + k;
    if (recs) write_records(a, Dv, recs, (int)(bg / Hk), (int)(bg % Hk), i, k, pos);
}

// The same two passes with the counts of a run of kIdxQueries queries first summed in
// shared memory (one counter per chunk): the global counters and cursors then take one
// atomic add per (CTA, chunk touched) instead of one per entry. Dynamic shared memory:
// C ints (count), 2 C ints (scatter). grid: (ceil(N / kIdxQueries), B * Hk).
constexpr int kIdxQueries = 256;
constexpr int kIdxThreads = 256;
constexpr int kIdxSmemMax = 96 * 1024;

__device__ __forceinline__ void run_histogram(const BwdAttendArgs &a, int64_t bg, int i0, int i1, int *hist) {
    const int K = a.topk, C = a.N / kChunk;
    for (int c = threadIdx.x; c < C; c += kIdxThreads) hist[c] = 0;
    __syncthreads();
    for (int64_t e = (bg * a.N + i0) * K + threadIdx.x; e < (bg * a.N + i1) * K; e += kIdxThreads) {
        const int64_t qg = e / K;
        const int k = (int)(e - qg * K);
        if (k >= min(max(a.nsel[qg], 0), K)) continue;
        const int c = a.idx[e];
        if (c >= 0 && c < C) atomicAdd(&hist[c], 1);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kIdxThreads) bwd_count_runs_kernel(BwdAttendArgs a, int *count) {
    extern __shared__ int hist[];
    const int C = a.N / kChunk;
    const int64_t bg = blockIdx.y;
    const int i0 = blockIdx.x * kIdxQueries, i1 = min(a.N, i0 + kIdxQueries);
    run_histogram(a, bg, i0, i1, hist);
    for (int c = threadIdx.x; c < C; c += kIdxThreads)
        if (hist[c]) atomicAdd(&count[bg * C + c], hist[c]);
}

__global__ void __launch_bounds__(kIdxThreads) bwd_scatter_runs_kernel(BwdAttendArgs a, int *cursor, int *entries,
                                                                       const float *Dv, int4 *recs) {
    extern __shared__ int hist[];  // [C] counts, then [C] this run's first positions
    const int C = a.N / kChunk, K = a.topk, Hk = a.H / a.G;
    int *base = hist + C;
    const int64_t bg = blockIdx.y;
    const int i0 = blockIdx.x * kIdxQueries, i1 = min(a.N, i0 + kIdxQueries);
    run_histogram(a, bg, i0, i1, hist);
    for (int c = threadIdx.x; c < C; c += kIdxThreads) {
        base[c] = hist[c] ? atomicAdd(&cursor[bg * C + c], hist[c]) : 0;
        hist[c] = 0;
    }
    __syncthreads();
    for (int64_t e = (bg * a.N + i0) * K + threadIdx.x; e < (bg * a.N + i1) * K; e += kIdxThreads) {
        const int64_t qg = e / K;
        const int k = (int)(e - qg * K);
        if (k >= min(max(a.nsel[qg], 0), K)) continue;
        const int c = a.idx[e];
        if (c < 0 || c >= C) continue;
        const int i = (int)(qg - bg * a.N);
        const int pos = base[c] + atomicAdd(&hist[c], 1);
        if (entries) entries[bg * (int64_t)a.N * K + pos] = i * 32 + k;
        if (recs) write_records(a, Dv, recs, (int)(bg / Hk), (int)(bg % Hk), i, k, pos);
    }
}

// Builds the group's inverted index (counts, starts and cursors; chunk items when `items`
// is given) and fills `entries` and/or `recs`.
hils_status build_index(const BwdAttendArgs &a, const BwdWs &w, int *entries, int4 *recs, int4 *items, int *nitems,
                        int max_items, cudaStream_t s) {
    const int Hk = a.H / a.G, C = a.N / kChunk;
    hils_status st = record_cuda_error(cudaMemsetAsync(w.count, 0, (size_t)a.B * Hk * C * sizeof(int), s));
    if (st != HILS_OK) return st;
    const size_t smem = (size_t)2 * C * sizeof(int);
    if (smem <= (size_t)kIdxSmemMax) {
        static KernelSetup setup_c, setup_s;
        st = kernel_setup(setup_c, (const void *)bwd_count_runs_kernel, kIdxThreads, kIdxSmemMax / 2, nullptr);
        if (st != HILS_OK) return st;
        st = kernel_setup(setup_s, (const void *)bwd_scatter_runs_kernel, kIdxThreads, kIdxSmemMax, nullptr);
        if (st != HILS_OK) return st;
        const dim3 grid((a.N + kIdxQueries - 1) / kIdxQueries, a.B * Hk);
        bwd_count_runs_kernel<<<grid, kIdxThreads, smem / 2, s>>>(a, w.count);
        bwd_scan_kernel<<<(unsigned)(a.B * Hk), 1024, 0, s>>>(C, w.count, w.start, w.cursor, items, nitems, max_items);
        bwd_scatter_runs_kernel<<<grid, kIdxThreads, smem, s>>>(a, w.cursor, entries, w.D, recs);
    } else {
        const int64_t ne = (int64_t)a.B * Hk * a.N * a.topk;
        bwd_count_kernel<<<(unsigned)((ne + 255) / 256), 256, 0, s>>>(a, w.count);
        bwd_scan_kernel<<<(unsigned)(a.B * Hk), 1024, 0, s>>>(C, w.count, w.start, w.cursor, items, nitems, max_items);
        bwd_scatter_kernel<<<(unsigned)((ne + 255) / 256), 256, 0, s>>>(a, w.cursor, entries, w.D, recs);
    }
    return record_cuda_error(cudaGetLastError());
}

constexpr int kQT = 16;  // queries per step of the key-major kernel

template <typename T, int D>
struct KmCfg {
    static constexpr int kLd = D + 1;  // padded row stride: column x of rows j in distinct banks
    // K and V rows of the block, the dk and dv accumulators ([64][kLd] float32 each), a
    // step's q and dO rows ([kQT][D]), their logits/dl and dO.v/cv ([kQT][64]), and the
    // step's per-query scalars
    static constexpr int kSmemBytes = (4 * kChunk * kLd + 2 * kQT * D + 2 * kQT * kChunk + 4 * kQT) * 4;
};

// One 64-key block of (b, h): window queries (kChunkMode = false) or the queries that
// kept chunk c (true), kQT at a time. grid: (key blocks or chunks, B * H).
template <typename T, int D, bool kChunkMode>
__global__ void __launch_bounds__(kThreads) attend_bwd_keymajor_kernel(BwdAttendArgs a, const float *Dv,
                                                                       const int *start, const int *entries) {
    using Cfg = KmCfg<T, D>;
    constexpr int kLd = Cfg::kLd;
    extern __shared__ __align__(16) float fsm[];
    float *kt = fsm, *vt = kt + kChunk * kLd, *dka = vt + kChunk * kLd, *dva = dka + kChunk * kLd;
    float *qs = dva + kChunk * kLd, *dos = qs + kQT * D;   // [kQT][D]
    float *lg = dos + kQT * D, *tj = lg + kQT * kChunk;    // [kQT][64]: logits -> dl, dO.v -> cv
    float *q_lse = tj + kQT * kChunk, *q_D = q_lse + kQT, *q_w = q_D + kQT;
    int *q_i = reinterpret_cast<int *>(q_w + kQT);
    const int tid = threadIdx.x;
    const int blk = blockIdx.x;
    const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int Hk = a.H / a.G, hk = h / a.G, K = a.topk, C = a.N / kChunk;
    const int j0 = blk * kChunk;
    const int rows = min(kChunk, a.N - j0);
    const T *kbase = static_cast<const T *>(a.K.ptr) + b * a.K.sb + hk * a.K.sh;
    const T *vbase = static_cast<const T *>(a.V.ptr) + b * a.V.sb + hk * a.V.sh;
    int q_begin, q_end;
    const int *list = nullptr;
    if (kChunkMode) {
        const int64_t bg = (int64_t)b * Hk + hk;
        q_begin = start[bg * (C + 1) + blk];
        q_end = start[bg * (C + 1) + blk + 1];
        list = entries + bg * (int64_t)a.N * K;
    } else {
        q_begin = j0;
        q_end = a.W > 0 ? min(a.N, j0 + rows - 1 + a.W) : j0;  // i with a window key in the block
    }
    if (q_begin >= q_end) return;
    for (int e = tid; e < kChunk * D; e += kThreads) {
        const int j = e / D, x = e - (e / D) * D;
        kt[j * kLd + x] = j < rows ? elem(kbase + (int64_t)(j0 + j) * a.K.st, x) : 0.f;
        vt[j * kLd + x] = j < rows ? elem(vbase + (int64_t)(j0 + j) * a.V.st, x) : 0.f;
        dka[j * kLd + x] = 0.f;
        dva[j * kLd + x] = 0.f;
    }
    const int64_t qhead = ((int64_t)b * a.H + h) * a.N;
    for (int q0 = q_begin; q0 < q_end; q0 += kQT) {
        const int nq = min(kQT, q_end - q0);
        __syncthreads();  // the previous step's rows and scalars are no longer read
        if (tid < kQT) {  // the step's queries: index, lse, D, and (chunks) slot k and score weight
            int i = -1, k = 0;
            float lse = -INFINITY, w = 0.f;
            if (tid < nq) {
                if (kChunkMode) {
                    const int en = list[q0 + tid];
                    i = en >> 5;
                    k = en & 31;
                } else {
                    i = q0 + tid;
                }
                lse = a.lse[qhead + i];
                if (kChunkMode && isfinite(lse)) w = expf(a.score[(qhead + i) * K + k] - lse);
            }
            q_i[tid] = isfinite(lse) ? (kChunkMode ? (i * 32 + k) : i) : -1;
            q_lse[tid] = lse;
            q_D[tid] = (i >= 0 && isfinite(lse)) ? Dv[qhead + i] : 0.f;
            q_w[tid] = w;
        }
        __syncthreads();
        for (int e = tid; e < kQT * D; e += kThreads) {
            const int r = e / D, x = e - (e / D) * D;
            const int en = q_i[r];
            const int i = en < 0 ? -1 : (kChunkMode ? en >> 5 : en);
            float qv = 0.f, dv = 0.f;
            if (i >= 0) {
                qv = elem(static_cast<const T *>(a.Q.ptr) + b * a.Q.sb + h * a.Q.sh + (int64_t)i * a.Q.st, x);
                dv = a.dO[(qhead + i) * D + x];
            }
            qs[e] = qv;
            dos[e] = dv;
        }
        __syncthreads();
        {  // logits l[r][j] = scale q_r . k_j and t[r][j] = dO_r . v_j: key j, queries r0..r0+7
            const int j = tid & (kChunk - 1), r0 = (tid >> 6) * (kQT / 2);
            float al[kQT / 2], at[kQT / 2];
#pragma unroll
            for (int r = 0; r < kQT / 2; ++r) al[r] = at[r] = 0.f;
            for (int x = 0; x < D; ++x) {
                const float kv = kt[j * kLd + x], vv = vt[j * kLd + x];
#pragma unroll
                for (int r = 0; r < kQT / 2; ++r) {
                    al[r] = fmaf(qs[(r0 + r) * D + x], kv, al[r]);
                    at[r] = fmaf(dos[(r0 + r) * D + x], vv, at[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < kQT / 2; ++r) {
                const int rr = r0 + r, en = q_i[rr];
                bool ok = en >= 0 && j < rows;
                if (!kChunkMode && ok) ok = j0 + j <= en && j0 + j > en - a.W;  // in query en's window
                lg[rr * kChunk + j] = ok ? al[r] * a.scale : -INFINITY;
                tj[rr * kChunk + j] = ok ? at[r] : 0.f;
            }
        }
        __syncthreads();
        {  // per query (a warp takes four): weights, dl (into lg) and cv (into tj), dscore
            const int lane = tid & 31, w = tid >> 5;
#pragma unroll
            for (int r4 = 0; r4 < kQT / 4; ++r4) {
                const int r = w * (kQT / 4) + r4;
                const int en = q_i[r];
                if (en < 0) {  // warp-uniform
                    lg[r * kChunk + lane] = lg[r * kChunk + lane + 32] = 0.f;
                    tj[r * kChunk + lane] = tj[r * kChunk + lane + 32] = 0.f;
                    continue;
                }
                const float l0 = lg[r * kChunk + lane], l1 = lg[r * kChunk + lane + 32];
                const float t0 = tj[r * kChunk + lane], t1 = tj[r * kChunk + lane + 32];
                const float Di = q_D[r];
                float d0, d1, c0, c1;
                if (kChunkMode) {
                    const float m = warp_max(fmaxf(l0, l1));
                    const float e0 = expf(l0 - m), e1 = expf(l1 - m);
                    const float inv = 1.f / warp_sum(e0 + e1);
                    const float p0 = e0 * inv, p1 = e1 * inv;
                    const float oc = warp_sum(p0 * t0 + p1 * t1);
                    const float wc = q_w[r];
                    d0 = wc * p0 * (t0 - oc);
                    d1 = wc * p1 * (t1 - oc);
                    c0 = wc * p0;
                    c1 = wc * p1;
                    if (lane == 0) a.dscore[(qhead + (en >> 5)) * K + (en & 31)] = wc * (oc - Di);
                } else {
                    const float lse = q_lse[r];
                    c0 = expf(l0 - lse);  // 0 outside the window
                    c1 = expf(l1 - lse);
                    d0 = c0 * (t0 - Di);
                    d1 = c1 * (t1 - Di);
                }
                lg[r * kChunk + lane] = d0;
                lg[r * kChunk + lane + 32] = d1;
                tj[r * kChunk + lane] = c0;
                tj[r * kChunk + lane + 32] = c1;
            }
        }
        __syncthreads();
        {  // dk_j += scale sum_r dl[r][j] q_r and dv_j += sum_r cv[r][j] dO_r: key j, a column half
            const int j = tid & (kChunk - 1), xh = (tid >> 6) * (D / 2);
            float dlr[kQT], cvr[kQT];
#pragma unroll
            for (int r = 0; r < kQT; ++r) {
                dlr[r] = a.scale * lg[r * kChunk + j];
                cvr[r] = tj[r * kChunk + j];
            }
            for (int x = xh; x < xh + D / 2; ++x) {
                float sk = dka[j * kLd + x], sv = dva[j * kLd + x];
#pragma unroll
                for (int r = 0; r < kQT; ++r) {
                    sk = fmaf(dlr[r], qs[r * D + x], sk);
                    sv = fmaf(cvr[r], dos[r * D + x], sv);
                }
                dka[j * kLd + x] = sk;
                dva[j * kLd + x] = sv;
            }
        }
        if (tid < D) {  // this block's share of dq_r: column tid
            float acc[kQT];
#pragma unroll
            for (int r = 0; r < kQT; ++r) acc[r] = 0.f;
            for (int j = 0; j < rows; ++j) {
                const float kv = kt[j * kLd + tid];
#pragma unroll
                for (int r = 0; r < kQT; ++r) acc[r] = fmaf(lg[r * kChunk + j], kv, acc[r]);
            }
            for (int r = 0; r < nq; ++r) {
                const int en = q_i[r];
                if (en < 0) continue;
                const int i = kChunkMode ? en >> 5 : en;
                atomicAdd(a.dQ + (qhead + i) * D + tid, a.scale * acc[r]);
            }
        }
    }
    __syncthreads();
    float *dkb = a.dK + ((int64_t)b * Hk + hk) * a.N * D + (int64_t)j0 * D;
    float *dvb = a.dV + ((int64_t)b * Hk + hk) * a.N * D + (int64_t)j0 * D;
    for (int e = tid; e < rows * D; e += kThreads) {
        const int j = e / D, x = e - (e / D) * D;
        atomicAdd(dkb + e, dka[j * kLd + x]);
        atomicAdd(dvb + e, dva[j * kLd + x]);
    }
}

// ---- the same key-major walk on the tensor cores (bf16 inputs): per step of 16 queries
// the products S = Q K^T and T = dO V^T (16 x 64), dK += dl^T Q, dV += cv^T dO (64 x d)
// and dQ += dl K (16 x d) are mma.sync m16n8k16 bf16 tiles with float32 accumulation; dO,
// dl and cv enter them rounded to bf16. Warp w owns keys 16w..16w+15 of the block (its
// dK and dV rows stay in registers for the whole walk) and a quarter of dQ's columns.

__device__ __forceinline__ void bw_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void bw_ldsm4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void bw_ldsm4t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

template <int D>
struct MmaCfg {
    static constexpr int kLds = D + 8;       // bf16 row stride of K, V, Q, dO (rows 16 B apart mod 128)
    static constexpr int kLdp = kChunk + 8;  // bf16 row stride of dl and cv
    static constexpr int kSmemBytes =
        (2 * kChunk * kLds + 2 * kQT * kLds + 2 * kQT * kLdp) * 2 + 2 * kQT * kChunk * 4 + 4 * kQT * 4;
};

template <int D, bool kChunkMode>
__global__ void __launch_bounds__(kThreads) attend_bwd_mma_kernel(BwdAttendArgs a, const float *Dv,
                                                                  const int *start, const int *entries) {
    using Cfg = MmaCfg<D>;
    constexpr int kLds = Cfg::kLds, kLdp = Cfg::kLdp, kNT = D / 8;
    extern __shared__ __align__(16) uint8_t bsm[];
    bf16 *kb = reinterpret_cast<bf16 *>(bsm), *vb = kb + kChunk * kLds;
    bf16 *qb = vb + kChunk * kLds, *dob = qb + kQT * kLds;
    bf16 *dlb = dob + kQT * kLds, *cvb = dlb + kQT * kLdp;             // [kQT][kLdp]
    float *lg = reinterpret_cast<float *>(cvb + kQT * kLdp), *tj = lg + kQT * kChunk;  // [kQT][64]
    float *q_lse = tj + kQT * kChunk, *q_D = q_lse + kQT, *q_w = q_D + kQT;
    int *q_i = reinterpret_cast<int *>(q_w + kQT);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t4 = lane & 3;
    const int blk = blockIdx.x;
    const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int Hk = a.H / a.G, hk = h / a.G, K = a.topk, C = a.N / kChunk;
    const int j0 = blk * kChunk;
    const int rows = min(kChunk, a.N - j0);
    const bf16 *kbase = static_cast<const bf16 *>(a.K.ptr) + b * a.K.sb + hk * a.K.sh;
    const bf16 *vbase = static_cast<const bf16 *>(a.V.ptr) + b * a.V.sb + hk * a.V.sh;
    int q_begin, q_end;
    const int *list = nullptr;
    if (kChunkMode) {
        const int64_t bg = (int64_t)b * Hk + hk;
        q_begin = start[bg * (C + 1) + blk];
        q_end = start[bg * (C + 1) + blk + 1];
        list = entries + bg * (int64_t)a.N * K;
    } else {
        q_begin = j0;
        q_end = a.W > 0 ? min(a.N, j0 + rows - 1 + a.W) : j0;
    }
    if (q_begin >= q_end) return;
    for (int e = tid; e < kChunk * D; e += kThreads) {
        const int j = e / D, x = e - (e / D) * D;
        const bf16 z = __float2bfloat16(0.f);
        kb[j * kLds + x] = j < rows ? kbase[(int64_t)(j0 + j) * a.K.st + x] : z;
        vb[j * kLds + x] = j < rows ? vbase[(int64_t)(j0 + j) * a.V.st + x] : z;
    }
    float dka[kNT][4], dva[kNT][4];  // this warp's 16 keys x D columns
#pragma unroll
    for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int r = 0; r < 4; ++r) dka[n][r] = dva[n][r] = 0.f;
    const int64_t qhead = ((int64_t)b * a.H + h) * a.N;
    for (int q0 = q_begin; q0 < q_end; q0 += kQT) {
        const int nq = min(kQT, q_end - q0);
        __syncthreads();
        if (tid < kQT) {
            int i = -1, k = 0;
            float lse = -INFINITY, w = 0.f;
            if (tid < nq) {
                if (kChunkMode) {
                    const int en = list[q0 + tid];
                    i = en >> 5;
                    k = en & 31;
                } else {
                    i = q0 + tid;
                }
                lse = a.lse[qhead + i];
                if (kChunkMode && isfinite(lse)) w = expf(a.score[(qhead + i) * K + k] - lse);
            }
            q_i[tid] = isfinite(lse) ? (kChunkMode ? (i * 32 + k) : i) : -1;
            q_lse[tid] = lse;
            q_D[tid] = (i >= 0 && isfinite(lse)) ? Dv[qhead + i] : 0.f;
            q_w[tid] = w;
        }
        __syncthreads();
        for (int e = tid; e < kQT * D; e += kThreads) {
            const int r = e / D, x = e - (e / D) * D;
            const int en = q_i[r];
            const int i = en < 0 ? -1 : (kChunkMode ? en >> 5 : en);
            bf16 qv = __float2bfloat16(0.f), dv = qv;
            if (i >= 0) {
                qv = static_cast<const bf16 *>(a.Q.ptr)[b * a.Q.sb + h * a.Q.sh + (int64_t)i * a.Q.st + x];
                dv = __float2bfloat16(a.dO[(qhead + i) * D + x]);
            }
            qb[r * kLds + x] = qv;
            dob[r * kLds + x] = dv;
        }
        __syncthreads();
        {  // S = Q K^T and T = dO V^T for this warp's 16 keys (two n-tiles of 8)
            float sa[2][4] = {}, ta[2][4] = {};
            const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t qa[4], da[4], kf[4], vf[4];
                const int arow = rr + (mi & 1) * 8, acol = ks * 16 + (mi >> 1) * 8;
                bw_ldsm4(qa, qb + arow * kLds + acol);
                bw_ldsm4(da, dob + arow * kLds + acol);
                const int brow = warp * 16 + (mi >> 1) * 8 + rr, bcol = ks * 16 + (mi & 1) * 8;
                bw_ldsm4(kf, kb + brow * kLds + bcol);
                bw_ldsm4(vf, vb + brow * kLds + bcol);
                bw_mma(sa[0], qa, kf[0], kf[1]);
                bw_mma(sa[1], qa, kf[2], kf[3]);
                bw_mma(ta[0], da, vf[0], vf[1]);
                bw_mma(ta[1], da, vf[2], vf[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hv = 0; hv < 2; ++hv)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int r = g + hv * 8, j = warp * 16 + nt * 8 + 2 * t4 + c;
                        const int en = q_i[r];
                        bool ok = en >= 0 && j < rows;
                        if (!kChunkMode && ok) ok = j0 + j <= en && j0 + j > en - a.W;
                        lg[r * kChunk + j] = ok ? sa[nt][hv * 2 + c] * a.scale : -INFINITY;
                        tj[r * kChunk + j] = ok ? ta[nt][hv * 2 + c] : 0.f;
                    }
        }
        __syncthreads();
        {  // per query (a warp takes four): weights, scale * dl and cv as bf16, dscore
#pragma unroll
            for (int r4 = 0; r4 < kQT / 4; ++r4) {
                const int r = warp * (kQT / 4) + r4;
                const int en = q_i[r];
                float d0 = 0.f, d1 = 0.f, c0 = 0.f, c1 = 0.f;
                if (en >= 0) {  // warp-uniform
                    const float l0 = lg[r * kChunk + lane], l1 = lg[r * kChunk + lane + 32];
                    const float t0 = tj[r * kChunk + lane], t1 = tj[r * kChunk + lane + 32];
                    const float Di = q_D[r];
                    if (kChunkMode) {
                        const float m = warp_max(fmaxf(l0, l1));
                        const float e0 = expf(l0 - m), e1 = expf(l1 - m);
                        const float inv = 1.f / warp_sum(e0 + e1);
                        const float p0 = e0 * inv, p1 = e1 * inv;
                        const float oc = warp_sum(p0 * t0 + p1 * t1);
                        const float wc = q_w[r];
                        d0 = wc * p0 * (t0 - oc);
                        d1 = wc * p1 * (t1 - oc);
                        c0 = wc * p0;
                        c1 = wc * p1;
                        if (lane == 0) a.dscore[(qhead + (en >> 5)) * K + (en & 31)] = wc * (oc - Di);
                    } else {
                        const float lse = q_lse[r];
                        c0 = expf(l0 - lse);
                        c1 = expf(l1 - lse);
                        d0 = c0 * (t0 - Di);
                        d1 = c1 * (t1 - Di);
                    }
                }
                dlb[r * kLdp + lane] = __float2bfloat16(a.scale * d0);
                dlb[r * kLdp + lane + 32] = __float2bfloat16(a.scale * d1);
                cvb[r * kLdp + lane] = __float2bfloat16(c0);
                cvb[r * kLdp + lane + 32] = __float2bfloat16(c1);
            }
        }
        __syncthreads();
        {  // dK += (scale dl)^T Q and dV += cv^T dO for this warp's keys: A = dl^T from the
           // [query][key] array (transposed load), B = Q / dO rows (transposed load)
            const int mi = lane >> 3, rr = lane & 7;
            uint32_t af[4], cf[4];
            const int arow = rr + (mi >> 1) * 8, acol = warp * 16 + (mi & 1) * 8;
            bw_ldsm4t(af, dlb + arow * kLdp + acol);
            bw_ldsm4t(cf, cvb + arow * kLdp + acol);
#pragma unroll
            for (int n2 = 0; n2 < kNT / 2; ++n2) {
                uint32_t qf4[4], df4[4];
                const int brow = rr + (mi & 1) * 8, bcol = n2 * 16 + (mi >> 1) * 8;
                bw_ldsm4t(qf4, qb + brow * kLds + bcol);
                bw_ldsm4t(df4, dob + brow * kLds + bcol);
                bw_mma(dka[2 * n2], af, qf4[0], qf4[1]);
                bw_mma(dka[2 * n2 + 1], af, qf4[2], qf4[3]);
                bw_mma(dva[2 * n2], cf, df4[0], df4[1]);
                bw_mma(dva[2 * n2 + 1], cf, df4[2], df4[3]);
            }
        }
        {  // dQ share: (scale dl) K for this warp's quarter of the columns
            constexpr int kWn = kNT / 4;  // n-tiles per warp
            float qa2[kWn][4] = {};
            const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
            for (int ks = 0; ks < kChunk / 16; ++ks) {
                uint32_t af[4];
                bw_ldsm4(af, dlb + (rr + (mi & 1) * 8) * kLdp + ks * 16 + (mi >> 1) * 8);
#pragma unroll
                for (int n2 = 0; n2 < kWn; n2 += 2) {
                    uint32_t kf4[4];
                    const int ncol = warp * kWn * 8 + n2 * 8;
                    bw_ldsm4t(kf4, kb + (ks * 16 + rr + (mi & 1) * 8) * kLds + ncol + (mi >> 1) * 8);
                    bw_mma(qa2[n2], af, kf4[0], kf4[1]);
                    if (n2 + 1 < kWn) bw_mma(qa2[n2 + 1], af, kf4[2], kf4[3]);
                }
            }
#pragma unroll
            for (int n = 0; n < kWn; ++n)
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {
                    const int r = g + hv * 8, en = q_i[r];
                    if (en < 0) continue;
                    const int i = kChunkMode ? en >> 5 : en;
                    float *dst = a.dQ + (qhead + i) * D + warp * kWn * 8 + n * 8 + 2 * t4;
                    atomicAdd(dst, qa2[n][hv * 2]);
                    atomicAdd(dst + 1, qa2[n][hv * 2 + 1]);
                }
        }
    }
    // this warp's keys' dK and dV into the global arrays
    float *dkb = a.dK + ((int64_t)b * Hk + hk) * a.N * D;
    float *dvb = a.dV + ((int64_t)b * Hk + hk) * a.N * D;
#pragma unroll
    for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
            const int j = warp * 16 + g + hv * 8;
            if (j >= rows) continue;
            float *pk = dkb + (int64_t)(j0 + j) * D + n * 8 + 2 * t4;
            float *pv = dvb + (int64_t)(j0 + j) * D + n * 8 + 2 * t4;
            atomicAdd(pk, dka[n][hv * 2]);
            atomicAdd(pk + 1, dka[n][hv * 2 + 1]);
            atomicAdd(pv, dva[n][hv * 2]);
            atomicAdd(pv + 1, dva[n][hv * 2 + 1]);
        }
}

// Eq. 7 backward, a CTA per kSelBwdRows consecutive queries of one (b, h):
//   1. dQcal = scale sum_k ds_k k'_{c_k}, a warp per query, the k' rows read from a copy
//      of the head's table in shared memory (or from global memory when it does not
//      fit); the kept entries are counted per chunk meanwhile;
//   2. the entries are sorted by chunk in shared memory (counting sort: a scan of the
//      counts, then each entry's slot from a cursor), as (query, ds) pairs;
//   3. warp w sums the entries of chunks c = w (mod 8) in registers, scale ds q~ over the
//      chunk's queries (eight q~ rows in flight) and ds for b', and adds the sums to dKsum
//      and dBsum once per (CTA, chunk) (vector atomics when dKsum is aligned).
// Used when the k' copy, the counts and the entries fit in shared memory.
constexpr int kSelBwdRows = 256;
constexpr int kSelBwdThreads = 256;
constexpr int kSelBwdWarps = kSelBwdThreads / 32;
constexpr int kSelBwdSmemMax = 200 * 1024;

// shared memory of the table kernel: counts / cursors [C], starts [C + 1], entries
// [kSelBwdRows * K] (query, ds), then (stage) the k' table [C][D]
__host__ __device__ inline size_t select_bwd_sort_bytes(int C, int K) {
    return ((size_t)(2 * C + 1) * 4 + 15) / 16 * 16 + (size_t)kSelBwdRows * (K > 0 ? K : 1) * 8;
}
template <typename T>
inline size_t select_bwd_smem_bytes(int C, int D, int K, bool stage) {
    return select_bwd_sort_bytes(C, K) + (stage ? (size_t)C * D * sizeof(T) : 0);
}

// E consecutive elements of a T row starting at element x, as floats (one vector load)
template <int E>
__device__ __forceinline__ void load_run(const bf16 *p, int x, float (&v)[E]) {
    if constexpr (E == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p + x);
        v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p + x);
        v[0] = bf16lo(u); v[1] = bf16hi(u);
    }
}
template <int E>
__device__ __forceinline__ void load_run(const float *p, int x, float (&v)[E]) {
    if constexpr (E == 4) {
        const float4 u = *reinterpret_cast<const float4 *>(p + x);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    } else {
        const float2 u = *reinterpret_cast<const float2 *>(p + x);
        v[0] = u.x; v[1] = u.y;
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kSelBwdThreads) select_backward_table_kernel(BwdSelectArgs a, int stage, int vec) {
    extern __shared__ __align__(16) uint8_t ssm[];
    constexpr int kE = D / 32;  // consecutive elements of a row per lane: 4 (D = 128) or 2
    const int C = a.C, K = a.topk;
    int *cnt = reinterpret_cast<int *>(ssm);  // [C] counts, then cursors
    int *off = cnt + C;                       // [C + 1] starts
    int2 *ent = reinterpret_cast<int2 *>(ssm + ((size_t)(2 * C + 1) * 4 + 15) / 16 * 16);  // (query, ds)
    T *ks = reinterpret_cast<T *>(ssm + select_bwd_sort_bytes(C, K));                        // [C][D]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nblk = (a.Lq + kSelBwdRows - 1) / kSelBwdRows;
    const int64_t bh = blockIdx.x / nblk;
    const int i0 = (int)(blockIdx.x % nblk) * kSelBwdRows;
    const int h = (int)(bh % a.H), b = (int)(bh / a.H);
    const int Hk = a.H / a.G;
    const T *khead = static_cast<const T *>(a.Ksum.ptr) + b * a.Ksum.sb + h * a.Ksum.sh;
    const T *qhead = static_cast<const T *>(a.Qcal.ptr) + b * a.Qcal.sb + h * a.Qcal.sh;
    for (int e = tid; e < C; e += kSelBwdThreads) cnt[e] = 0;
    if (stage) {  // the head's k' rows, 16 bytes per copy
        constexpr int kU = D * (int)sizeof(T) / 16;  // 16-byte units per row
        for (int e = tid; e < C * kU; e += kSelBwdThreads) {
            const int c = e / kU, u = e - c * kU;
            reinterpret_cast<uint4 *>(ks + (int64_t)c * D)[u] =
                reinterpret_cast<const uint4 *>(khead + (int64_t)c * a.Ksum.st)[u];
        }
    }
    __syncthreads();
    const T *kbase = stage ? ks : khead;
    const int64_t kst = stage ? D : a.Ksum.st;
    const int iend = min(a.Lq, i0 + kSelBwdRows);
    // lane k < K: kept chunk k's index and gradient (c = -1 when not kept)
    auto load_list = [&](int i, int &c, float &ds) {
        c = -1;
        ds = 0.f;
        if (i >= iend || lane >= K) return;
        const int64_t qg = ((int64_t)b * Hk + h / a.G) * a.Lq + i;
        const int ns = min(max(__ldg(&a.nsel[qg]), 0), K);
        const int cc = __ldg(&a.idx[qg * K + lane]);
        const float d = __ldg(&a.dscore[(bh * a.Lq + i) * K + lane]);
        if (lane < ns && (unsigned)cc < (unsigned)C) {
            c = cc;
            ds = d;
        }
    };
    // ---- 1. dQcal, a warp per query; counts per chunk
    {
        int myc, nc;
        float myds, nd;
        load_list(i0 + warp, myc, myds);
        for (int i = i0 + warp; i < iend; i += kSelBwdWarps) {
            load_list(i + kSelBwdWarps, nc, nd);  // the next query's list, in flight meanwhile
            if (myc >= 0) atomicAdd(&cnt[myc], 1);
            float acc[kE] = {};
            unsigned m = __ballot_sync(kFull, myc >= 0);
            while (m) {
                const int k = __ffs(m) - 1;
                m &= m - 1;
                const int c = __shfl_sync(kFull, myc, k);
                const float ds = __shfl_sync(kFull, myds, k);
                float kv[kE];
                load_run<kE>(kbase + (int64_t)c * kst, kE * lane, kv);
#pragma unroll
                for (int u = 0; u < kE; ++u) acc[u] = fmaf(ds, kv[u], acc[u]);
            }
            float *dq = a.dQcal + (bh * a.Lq + i) * D + kE * lane;
#pragma unroll
            for (int u = 0; u < kE; ++u) dq[u] = a.scale * acc[u];
            myc = nc;
            myds = nd;
        }
    }
    __syncthreads();
    // ---- 2. starts (exclusive scan of the counts, warp 0), cursors, then each entry's slot
    if (warp == 0) {
        int run = 0;
        for (int c0 = 0; c0 < C; c0 += 32) {
            const int c = c0 + lane;
            const int v = c < C ? cnt[c] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += u;
            }
            if (c < C) {
                off[c] = run + incl - v;
                cnt[c] = run + incl - v;
            }
            run += __shfl_sync(kFull, incl, 31);
        }
        if (lane == 0) off[C] = run;
    }
    __syncthreads();
    for (int i = i0 + warp; i < iend; i += kSelBwdWarps) {
        int c;
        float ds;
        load_list(i, c, ds);
        if (c >= 0) ent[atomicAdd(&cnt[c], 1)] = make_int2(i, __float_as_int(ds));
    }
    __syncthreads();
    // ---- 3. chunk sums of this warp's chunks, in registers
    float *dks = a.dKsum + bh * C * D;
    float *dbs = a.dBsum + bh * C;
    for (int c = warp; c < C; c += kSelBwdWarps) {
        const int e0 = off[c], e1 = off[c + 1];
        if (e0 == e1) continue;
        float acc[kE] = {};
        float db = 0.f;
        for (int e = e0; e < e1; e += 8) {
            float q[8][kE], dsv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {  // eight rows in flight
                const int2 en = ent[min(e + k, e1 - 1)];
                dsv[k] = e + k < e1 ? __int_as_float(en.y) : 0.f;
                load_run<kE>(qhead + (int64_t)en.x * a.Qcal.st, kE * lane, q[k]);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                db += dsv[k];
#pragma unroll
                for (int u = 0; u < kE; ++u) acc[u] = fmaf(dsv[k], q[k][u], acc[u]);
            }
        }
        float *dst = dks + (int64_t)c * D + kE * lane;
#pragma unroll
        for (int u = 0; u < kE; ++u) acc[u] *= a.scale;
        if (vec) {
            if constexpr (kE == 4) atomicAdd(reinterpret_cast<float4 *>(dst), make_float4(acc[0], acc[1], acc[2], acc[3]));
            else atomicAdd(reinterpret_cast<float2 *>(dst), make_float2(acc[0], acc[1]));
        } else {
#pragma unroll
            for (int u = 0; u < kE; ++u) atomicAdd(dst + u, acc[u]);
        }
        if (lane == 0) atomicAdd(dbs + c, db);
    }
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
hils_status launch_attend_bwd(const BwdAttendArgs &a, void *ws, cudaStream_t s) {
    const int64_t nq = (int64_t)a.B * a.H * a.N;
    const int Hk = a.H / a.G, C = a.N / kChunk;
    constexpr bool kTc = sizeof(T) == 2 && D == 128;
    const BwdWs w = bwd_ws(ws, kTc, a.B, a.H, Hk, a.N, a.topk, D);
    hils_status st = record_cuda_error(cudaMemsetAsync(w.status, 0, sizeof(uint32_t), s));
    if (st != HILS_OK) return st;
    st = record_cuda_error(cudaMemsetAsync(a.dQ, 0, (size_t)nq * D * sizeof(float), s));
    if (st != HILS_OK) return st;
    if (a.topk > 0) {  // dscore padding stays 0
        st = record_cuda_error(cudaMemsetAsync(a.dscore, 0, (size_t)nq * a.topk * sizeof(float), s));
        if (st != HILS_OK) return st;
    }
    if constexpr (kTc) {
        // tensor-core walk: D_i and the contiguous bf16 rows, the inverted index with its
        // per-head records and chunk items, then one launch over all work items
        bwd_prep_kernel<<<(unsigned)((nq + 3) / 4), kThreads, 0, s>>>(a, w.D, w.dOb, w.Qc);
        const bool chunks = a.topk > 0 && C > 0;
        if (chunks) {
            st = build_index(a, w, nullptr, w.recs, w.items, w.nitems, w.max_items, s);
            if (st != HILS_OK) return st;
        }
        BwdTcArgs t;
        t.a = a;
        t.Dv = w.D;
        t.recs = w.recs;
        t.items = w.items;
        t.nitems = w.nitems;
        t.max_items = chunks ? w.max_items : 0;
        t.nsegw = a.W > 0 ? (kChunk - 1 + a.W + kBwdItemQueries - 1) / kBwdItemQueries : 0;
        t.nwin = a.W > 0 ? ((a.N + kChunk - 1) / kChunk) * t.nsegw : 0;
        t.vec_ok = ((uintptr_t)a.dQ & 15u) == 0;
        t.status = w.status;
        st = record_cuda_error(cudaGetLastError());
        if (st != HILS_OK) return st;
        return launch_attend_bwd_tc(t, w.Qc, w.dOb, s);
    } else {
        bwd_dot_kernel<T, D><<<(unsigned)((nq + 3) / 4), kThreads, 0, s>>>(a, w.D);
        // bf16, d = 64: the mma.sync walk; float32: the CUDA-core walk (full float32 products)
        constexpr bool kMma = sizeof(T) == 2;
        constexpr int smem = kMma ? MmaCfg<D>::kSmemBytes : KmCfg<T, D>::kSmemBytes;
        const void *fw = kMma ? (const void *)attend_bwd_mma_kernel<D, false>
                              : (const void *)attend_bwd_keymajor_kernel<T, D, false>;
        const void *fc = kMma ? (const void *)attend_bwd_mma_kernel<D, true>
                              : (const void *)attend_bwd_keymajor_kernel<T, D, true>;
        static KernelSetup setup_w, setup_c;
        st = kernel_setup(setup_w, fw, kThreads, smem, nullptr);
        if (st != HILS_OK) return st;
        st = kernel_setup(setup_c, fc, kThreads, smem, nullptr);
        if (st != HILS_OK) return st;
        if (a.topk > 0 && C > 0) {
            st = build_index(a, w, w.entries, nullptr, nullptr, nullptr, 0, s);
            if (st != HILS_OK) return st;
            if constexpr (kMma)
                attend_bwd_mma_kernel<D, true><<<dim3(C, a.B * a.H), kThreads, smem, s>>>(a, w.D, w.start, w.entries);
            else
                attend_bwd_keymajor_kernel<T, D, true><<<dim3(C, a.B * a.H), kThreads, smem, s>>>(a, w.D, w.start,
                                                                                                    w.entries);
        }
        if (a.W > 0) {
            const dim3 grid((a.N + kChunk - 1) / kChunk, a.B * a.H);
            if constexpr (kMma) attend_bwd_mma_kernel<D, false><<<grid, kThreads, smem, s>>>(a, w.D, nullptr, nullptr);
            else attend_bwd_keymajor_kernel<T, D, false><<<grid, kThreads, smem, s>>>(a, w.D, nullptr, nullptr);
        }
        return record_cuda_error(cudaGetLastError());
    }
}

template <typename T, int D>
hils_status launch_select_bwd(const BwdSelectArgs &a, cudaStream_t s) {
    // the per-chunk counts and starts and the CTA's entries must fit in shared memory:
    // C up to about 21,000 chunks (1.3M tokens) at K = 16
    if (a.C > 0 && select_bwd_smem_bytes<T>(a.C, D, a.topk, false) <= (size_t)kSelBwdSmemMax) {
        const bool stage = select_bwd_smem_bytes<T>(a.C, D, a.topk, true) <= (size_t)kSelBwdSmemMax;
        const size_t smem = select_bwd_smem_bytes<T>(a.C, D, a.topk, stage);
        // dKsum rows start 16 (D = 128) or 8 (D = 64) bytes apart from an aligned base
        const int vec = ((uintptr_t)a.dKsum & (D == 128 ? 15u : 7u)) == 0;
        static KernelSetup setup;
        const hils_status st = kernel_setup(setup, (const void *)select_backward_table_kernel<T, D>, kSelBwdThreads,
                                            kSelBwdSmemMax, nullptr);
        if (st != HILS_OK) return st;
        const int64_t grid = (int64_t)a.B * a.H * ((a.Lq + kSelBwdRows - 1) / kSelBwdRows);
        select_backward_table_kernel<T, D><<<(unsigned)grid, kSelBwdThreads, smem, s>>>(a, stage ? 1 : 0, vec);
        return record_cuda_error(cudaGetLastError());
    }
    if (a.C > 0) return HILS_ERR_UNSUPPORTED;
    // no summarised chunk: nothing was kept, dQcal is zero
    return record_cuda_error(cudaMemsetAsync(a.dQcal, 0, (size_t)a.B * a.H * a.Lq * D * sizeof(float), s));
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

hils_status launch_attend_backward(hils_dtype dt, int d, const BwdAttendArgs &a, void *ws, cudaStream_t s) {
    if ((int64_t)a.B * a.H * a.N == 0) return HILS_OK;
    if (dt == HILS_BF16)
        return d == 64 ? launch_attend_bwd<bf16, 64>(a, ws, s) : launch_attend_bwd<bf16, 128>(a, ws, s);
    return d == 64 ? launch_attend_bwd<float, 64>(a, ws, s) : launch_attend_bwd<float, 128>(a, ws, s);
}

size_t attend_backward_ws_bytes(hils_dtype dt, int d, int B, int H, int Hk, int N, int K) {
    return bwd_ws(nullptr, bwd_tc_layout(dt, d), B, H, Hk, N, K, d).bytes;
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
