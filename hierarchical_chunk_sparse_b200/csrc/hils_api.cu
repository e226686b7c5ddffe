// C-ABI entry points of libhils: argument validation, workspace sizing and dispatch
// to one kernel launcher per stage. No call allocates, frees or synchronises.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "backward_common.cuh"
#include "hils_internal.cuh"

namespace hils {

static thread_local char g_last_error[256] = "";

hils_status record_cuda_error(cudaError_t e) {
    if (e == cudaSuccess) return HILS_OK;
    snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return HILS_ERR_CUDA;
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 1;
    return n;
}

hils_status kernel_setup(KernelSetup &cache, const void *func, int threads, int smem_bytes, int *per_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return record_cuda_error(e);
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (__atomic_load_n(&cache.done, __ATOMIC_ACQUIRE) & bit)) {
        if (per_sm) *per_sm = cache.per_sm[dev];
        return HILS_OK;
    }
    if (smem_bytes > 0) {  // also needed when static + dynamic shared memory passes 48 KB
        e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
        if (e != cudaSuccess) return record_cuda_error(e);
    }
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem_bytes);
    if (e != cudaSuccess) return record_cuda_error(e);
    if (n < 1) n = 1;
    if (bit) {
        cache.per_sm[dev] = n;
        __atomic_fetch_or(&cache.done, bit, __ATOMIC_RELEASE);
    }
    if (per_sm) *per_sm = n;
    return HILS_OK;
}

namespace {

size_t elem_size(hils_dtype dt) { return dt == HILS_BF16 ? 2 : 4; }

// Common parameter checks; fills the effective scale.
int check_params(const hils_params *p, float *scale) {
    if (!p) return HILS_ERR_INVALID_ARG;
    if (p->B < 0 || p->H < 0 || p->K < 0 || p->W < 0) return HILS_ERR_INVALID_ARG;
    if (p->dtype != HILS_F32 && p->dtype != HILS_BF16) return HILS_ERR_UNSUPPORTED;
    if (p->d != 64 && p->d != 128) return HILS_ERR_UNSUPPORTED;
    if (p->S != kChunk) return HILS_ERR_UNSUPPORTED;
    if (p->K > 32) return HILS_ERR_UNSUPPORTED;
    if (p->flags & ~(uint32_t)(HILS_FLAG_EXCLUDE_WINDOW_CHUNKS | HILS_FLAG_DIAG_EXPIRE_WAITS))
        return HILS_ERR_UNSUPPORTED;
    if (!isfinite(p->scale)) return HILS_ERR_INVALID_ARG;
    if (p->H_kv < 0 || (p->H_kv > 0 && p->H % p->H_kv != 0)) return HILS_ERR_INVALID_ARG;
    if (p->H_kv > 0 && p->H / p->H_kv > kMaxGroupHeads) return HILS_ERR_UNSUPPORTED;
    *scale = p->scale != 0.f ? p->scale : (float)(1.0 / sqrt((double)p->d));
    return HILS_OK;
}

// Query heads per key-value head (parameters already checked).
int groups(const hils_params *p) { return p->H_kv > 0 ? p->H / p->H_kv : 1; }

bool aligned16(const void *ptr) { return ((uintptr_t)ptr & 15u) == 0; }

// A [B, H, T, d] view with T rows used: non-null when it holds elements, 16-byte
// aligned base and strides.
int check_view(const void *ptr, int64_t sb, int64_t sh, int64_t st, int64_t rows, const hils_params *p) {
    if ((int64_t)p->B * p->H * rows == 0) return HILS_OK;
    if (!ptr) return HILS_ERR_INVALID_ARG;
    const int64_t es = (int64_t)elem_size(p->dtype);
    if (!aligned16(ptr)) return HILS_ERR_ALIGNMENT;
    if ((sb * es) % 16 || (sh * es) % 16 || (st * es) % 16) return HILS_ERR_ALIGNMENT;
    return HILS_OK;
}

int check_array(const void *ptr, int64_t count) {
    if (count > 0 && !ptr) return HILS_ERR_INVALID_ARG;
    if (ptr && ((uintptr_t)ptr & 3u)) return HILS_ERR_ALIGNMENT;
    return HILS_OK;
}

int check_workspace(const void *ws, size_t have, size_t need) {
    if (need == 0) return HILS_OK;
    if (!ws || have < need) return HILS_ERR_WORKSPACE;
    if (!aligned16(ws)) return HILS_ERR_ALIGNMENT;
    return HILS_OK;
}

// Units per query of the attend kernels: one per kept chunk plus the window tiles
// (at least one, so that an empty query still gets o = 0 and lse = -inf).
int decode_units(const hils_params *p) {
    const int u = p->K + (p->W + kChunk - 1) / kChunk;
    return u > 0 ? u : 1;
}

size_t select_ws_for(const hils_params *p, int Lq, int C) {
    SelectArgs a{};
    a.G = groups(p);
    select_plan(p->dtype, p->d, p->B, p->H, Lq, C, p->K, true, device_sm_count(), &a);
    return select_ws_bytes(p->B * p->H * Lq, C, a.path);
}

#define HILS_TRY(expr)                 \
    do {                               \
        const int _rc = (expr);        \
        if (_rc != HILS_OK) return _rc; \
    } while (0)


int prepare_select(const hils_params *p, hils_ctensor Qcal, int Lq, const int32_t *qpos, int qpos_bias,
                   hils_ctensor Ksum, const float *Bsum, int C, int32_t *idx, float *score, int32_t *nsel,
                   SelectArgs *a, int64_t *nq_out) {
    float scale;
    HILS_TRY(check_params(p, &scale));
    if (Lq < 0 || C < 0) return HILS_ERR_INVALID_ARG;
    const int64_t nq = (int64_t)p->B * p->H * Lq;
    if (nq > 0x7fffffffll) return HILS_ERR_INVALID_ARG;  // query count fits in int
    HILS_TRY(check_view(Qcal.ptr, Qcal.sb, Qcal.sh, Qcal.st, Lq, p));
    HILS_TRY(check_view(Ksum.ptr, Ksum.sb, Ksum.sh, Ksum.st, C, p));
    HILS_TRY(check_array(Bsum, (int64_t)p->B * p->H * C));
    HILS_TRY(check_array(idx, nq / groups(p) * p->K));
    HILS_TRY(check_array(score, nq * p->K));
    HILS_TRY(check_array(nsel, nq / groups(p)));
    if (qpos && ((uintptr_t)qpos & 3u)) return HILS_ERR_ALIGNMENT;
    *nq_out = nq;
    a->Qcal = {Qcal.ptr, Qcal.sb, Qcal.sh, Qcal.st};
    a->Ksum = {Ksum.ptr, Ksum.sb, Ksum.sh, Ksum.st};
    a->Bsum = Bsum;
    a->qpos = qpos;
    a->qpos_bias = qpos ? qpos_bias : 0;
    a->idx = idx;
    a->score = score;
    a->nsel = nsel;
    a->B = p->B;
    a->H = p->H;
    a->Lq = Lq;
    a->C = C;
    a->topk = p->K;
    a->scale = scale;
    a->G = groups(p);
    a->excl_w = (p->flags & HILS_FLAG_EXCLUDE_WINDOW_CHUNKS) ? p->W : 0;
    if (nq > 0) select_plan(p->dtype, p->d, p->B, p->H, Lq, C, p->K, qpos != nullptr, device_sm_count(), a);
    // the diagnostic expiry applies to the tensor-core select, which writes nothing after one
    a->wait_ns = a->path == kSelectTc ? work_wait_ns(p->flags) : kWaitLimitNs;
    return HILS_OK;
}

int prepare_attend_decode(const hils_params *p, hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc,
                          const int32_t *cache_len, const int32_t *idx, const float *score, const int32_t *nsel,
                          hils_tensor O, float *lse, AttendArgs *a) {
    float scale;
    HILS_TRY(check_params(p, &scale));
    const int64_t nq = (int64_t)p->B * p->H;
    HILS_TRY(check_view(Q.ptr, Q.sb, Q.sh, Q.st, 1, p));
    HILS_TRY(check_view(Kc.ptr, Kc.sb, Kc.sh, Kc.st, 1, p));
    HILS_TRY(check_view(Vc.ptr, Vc.sb, Vc.sh, Vc.st, 1, p));
    HILS_TRY(check_view(O.ptr, O.sb, O.sh, O.st, 1, p));
    HILS_TRY(check_array(cache_len, p->B));
    HILS_TRY(check_array(idx, nq / groups(p) * p->K));
    HILS_TRY(check_array(score, nq * p->K));
    HILS_TRY(check_array(nsel, p->K > 0 ? nq / groups(p) : 0));
    HILS_TRY(check_array(lse, 0));
    a->Q = {Q.ptr, Q.sb, Q.sh, Q.st};
    a->K = {Kc.ptr, Kc.sb, Kc.sh, Kc.st};
    a->V = {Vc.ptr, Vc.sb, Vc.sh, Vc.st};
    a->O = {O.ptr, O.sb, O.sh, O.st};
    a->lse = lse;
    a->idx = idx;
    a->score = score;
    a->nsel = nsel;
    a->qpos = nullptr;
    a->cache_len = cache_len;
    a->B = p->B;
    a->H = p->H;
    a->Lq = 1;
    a->topk = p->K;
    a->W = p->W;
    a->scale = scale;
    a->units = decode_units(p);
    a->G = groups(p);
    return HILS_OK;
}

}  // namespace

int check_attend_decode_args(const hils_params *p, hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc,
                             const int32_t *cache_len, const int32_t *idx, const float *score, const int32_t *nsel,
                             hils_tensor O, float *lse) {
    AttendArgs a{};
    return prepare_attend_decode(p, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse, &a);
}

namespace {

// The select part of a hils_decode workspace, rounded so the attend part starts aligned.
size_t decode_select_part(size_t select_bytes) { return (select_bytes + 255) & ~(size_t)255; }

}  // namespace
}  // namespace hils

using namespace hils;

extern "C" {

const char *hils_status_string(int status) {
    switch (status) {
    case HILS_OK: return "ok";
    case HILS_ERR_INVALID_ARG: return "invalid argument";
    case HILS_ERR_UNSUPPORTED: return "unsupported configuration (d in {64,128}, S = 64, K <= 32, known flags, H / H_kv <= 8)";
    case HILS_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case HILS_ERR_WORKSPACE: return "workspace missing or too small";
    case HILS_ERR_CUDA: return "CUDA launch error";
    default: return "unknown status";
    }
}

const char *hils_last_cuda_error(void) { return g_last_error; }

size_t hils_workspace_bytes(const hils_params *p, int call, int Lq, int C) {
    float scale;
    if (check_params(p, &scale) != HILS_OK || Lq < 0 || C < 0) return 0;
    switch (call) {
    case HILS_CALL_SELECT: return select_ws_for(p, Lq, C);
    case HILS_CALL_ATTEND_PREFILL: return kPrefillWsBytes;
    case HILS_CALL_ATTEND_DECODE: return attend_decode_ws_bytes(p->B * p->H, decode_units(p), p->d);
    case HILS_CALL_ATTEND_BACKWARD: return attend_backward_ws_bytes(p->dtype, p->d, p->B, p->H, p->H / groups(p), Lq, p->K);
    case HILS_CALL_DECODE:
        return decode_select_part(select_ws_for(p, 1, C)) + attend_decode_ws_bytes(p->B * p->H, decode_units(p), p->d);
    default: return 0;
    }
}

int hils_workspace_init(void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (ws_bytes == 0) return HILS_OK;
    if (!workspace) return HILS_ERR_INVALID_ARG;
    return record_cuda_error(cudaMemsetAsync(workspace, 0, ws_bytes, stream));
}

int hils_summarize(const hils_params *p, hils_ctensor K, int N, hils_ctensor LQ, hils_tensor Ksum,
                   float *Bsum, cudaStream_t stream) {
    float scale;
    HILS_TRY(check_params(p, &scale));
    if (N < 0) return HILS_ERR_INVALID_ARG;
    const int C = N / kChunk;
    if ((int64_t)p->B * p->H * C > 0xffffffffll) return HILS_ERR_INVALID_ARG;  // chunk count fits 32 bits
    HILS_TRY(check_view(K.ptr, K.sb, K.sh, K.st, (int64_t)C * kChunk, p));
    HILS_TRY(check_view(LQ.ptr, LQ.sb, LQ.sh, LQ.st, C, p));
    HILS_TRY(check_view(Ksum.ptr, Ksum.sb, Ksum.sh, Ksum.st, C, p));
    HILS_TRY(check_array(Bsum, (int64_t)p->B * p->H * C));
    SummarizeArgs a;
    a.K = {K.ptr, K.sb, K.sh, K.st};
    a.LQ = {LQ.ptr, LQ.sb, LQ.sh, LQ.st};
    a.Ksum = {Ksum.ptr, Ksum.sb, Ksum.sh, Ksum.st};
    a.Bsum = Bsum;
    a.B = p->B;
    a.H = p->H;
    a.C = C;
    a.scale = scale;
    a.G = groups(p);
    return launch_summarize(p->dtype, p->d, a, stream);
}

int hils_summarize_append(const hils_params *p, hils_ctensor K, const int32_t *cache_len, hils_ctensor LQ,
                          hils_tensor Ksum, float *Bsum, int C, cudaStream_t stream) {
    float scale;
    HILS_TRY(check_params(p, &scale));
    if (C < 0) return HILS_ERR_INVALID_ARG;
    if ((int64_t)p->B * p->H * C > 0xffffffffll) return HILS_ERR_INVALID_ARG;
    HILS_TRY(check_view(K.ptr, K.sb, K.sh, K.st, (int64_t)C * kChunk, p));
    HILS_TRY(check_view(LQ.ptr, LQ.sb, LQ.sh, LQ.st, C, p));
    HILS_TRY(check_view(Ksum.ptr, Ksum.sb, Ksum.sh, Ksum.st, C, p));
    HILS_TRY(check_array(Bsum, (int64_t)p->B * p->H * C));
    HILS_TRY(check_array(cache_len, C > 0 ? p->B : 0));
    SummarizeArgs a;
    a.K = {K.ptr, K.sb, K.sh, K.st};
    a.LQ = {LQ.ptr, LQ.sb, LQ.sh, LQ.st};
    a.Ksum = {Ksum.ptr, Ksum.sb, Ksum.sh, Ksum.st};
    a.Bsum = Bsum;
    a.B = p->B;
    a.H = p->H;
    a.C = C;
    a.scale = scale;
    a.G = groups(p);
    a.cache_len = cache_len;
    return launch_summarize(p->dtype, p->d, a, stream);
}

int hils_attend_prefill_backward(const hils_params *p, hils_ctensor Q, hils_ctensor K, hils_ctensor V, int N,
                                 const int32_t *idx, const float *score, const int32_t *nsel, hils_ctensor O,
                                 const float *lse, const float *dO, float *dQ, float *dK, float *dV, float *dscore,
                                 void *workspace, size_t ws_bytes, cudaStream_t stream) {
    float scale;
    HILS_TRY(check_params(p, &scale));
    if (N < 0) return HILS_ERR_INVALID_ARG;
    const int64_t nq = (int64_t)p->B * p->H * N;
    if (nq > 0x7fffffffll) return HILS_ERR_INVALID_ARG;
    const int64_t nkv = (int64_t)p->B * (p->H / groups(p)) * N * p->d;
    HILS_TRY(check_view(Q.ptr, Q.sb, Q.sh, Q.st, N, p));
    HILS_TRY(check_view(K.ptr, K.sb, K.sh, K.st, N, p));
    HILS_TRY(check_view(V.ptr, V.sb, V.sh, V.st, N, p));
    HILS_TRY(check_view(O.ptr, O.sb, O.sh, O.st, N, p));
    HILS_TRY(check_array(idx, nq / groups(p) * p->K));
    HILS_TRY(check_array(score, nq * p->K));
    HILS_TRY(check_array(nsel, p->K > 0 ? nq / groups(p) : 0));
    HILS_TRY(check_array(lse, nq));
    HILS_TRY(check_array(dO, nq * p->d));
    HILS_TRY(check_array(dQ, nq * p->d));
    HILS_TRY(check_array(dK, nkv));
    HILS_TRY(check_array(dV, nkv));
    HILS_TRY(check_array(dscore, nq * p->K));
    if (nq == 0) return HILS_OK;
    HILS_TRY(check_workspace(workspace, ws_bytes,
                             attend_backward_ws_bytes(p->dtype, p->d, p->B, p->H, p->H / groups(p), N, p->K)));
    BwdAttendArgs a;
    a.Q = {Q.ptr, Q.sb, Q.sh, Q.st};
    a.K = {K.ptr, K.sb, K.sh, K.st};
    a.V = {V.ptr, V.sb, V.sh, V.st};
    a.O = {O.ptr, O.sb, O.sh, O.st};
    a.lse = lse;
    a.dO = dO;
    a.score = score;
    a.idx = idx;
    a.nsel = nsel;
    a.dQ = dQ;
    a.dK = dK;
    a.dV = dV;
    a.dscore = dscore;
    a.B = p->B;
    a.H = p->H;
    a.N = N;
    a.topk = p->K;
    a.W = p->W;
    a.G = groups(p);
    a.scale = scale;
    a.wait_ns = work_wait_ns(p->flags);
    return launch_attend_backward(p->dtype, p->d, a, workspace, stream);
}

int hils_select_backward(const hils_params *p, hils_ctensor Qcal, int Lq, hils_ctensor Ksum, int C,
                         const int32_t *idx, const int32_t *nsel, const float *dscore, float *dQcal, float *dKsum,
                         float *dBsum, cudaStream_t stream) {
    float scale;
    HILS_TRY(check_params(p, &scale));
    if (Lq < 0 || C < 0) return HILS_ERR_INVALID_ARG;
    const int64_t nq = (int64_t)p->B * p->H * Lq;
    if (nq > 0x7fffffffll) return HILS_ERR_INVALID_ARG;
    HILS_TRY(check_view(Qcal.ptr, Qcal.sb, Qcal.sh, Qcal.st, Lq, p));
    HILS_TRY(check_view(Ksum.ptr, Ksum.sb, Ksum.sh, Ksum.st, C, p));
    HILS_TRY(check_array(idx, nq / groups(p) * p->K));
    HILS_TRY(check_array(nsel, p->K > 0 ? nq / groups(p) : 0));
    HILS_TRY(check_array(dscore, nq * p->K));
    HILS_TRY(check_array(dQcal, nq * p->d));
    HILS_TRY(check_array(dKsum, (int64_t)p->B * p->H * C * p->d));
    HILS_TRY(check_array(dBsum, (int64_t)p->B * p->H * C));
    BwdSelectArgs a;
    a.Qcal = {Qcal.ptr, Qcal.sb, Qcal.sh, Qcal.st};
    a.Ksum = {Ksum.ptr, Ksum.sb, Ksum.sh, Ksum.st};
    a.idx = idx;
    a.nsel = nsel;
    a.dscore = dscore;
    a.dQcal = dQcal;
    a.dKsum = dKsum;
    a.dBsum = dBsum;
    a.B = p->B;
    a.H = p->H;
    a.Lq = Lq;
    a.C = C;
    a.topk = p->K;
    a.G = groups(p);
    a.scale = scale;
    return launch_select_backward(p->dtype, p->d, a, stream);
}

int hils_summarize_backward(const hils_params *p, hils_ctensor K, int N, hils_ctensor LQ, const float *dKsum,
                            const float *dBsum, float *dK, float *dLQ, cudaStream_t stream) {
    float scale;
    HILS_TRY(check_params(p, &scale));
    if (N < 0) return HILS_ERR_INVALID_ARG;
    const int C = N / kChunk;
    if ((int64_t)p->B * p->H * C > 0x7fffffffll) return HILS_ERR_INVALID_ARG;
    HILS_TRY(check_view(K.ptr, K.sb, K.sh, K.st, (int64_t)C * kChunk, p));
    HILS_TRY(check_view(LQ.ptr, LQ.sb, LQ.sh, LQ.st, C, p));
    HILS_TRY(check_array(dKsum, (int64_t)p->B * p->H * C * p->d));
    HILS_TRY(check_array(dBsum, (int64_t)p->B * p->H * C));
    HILS_TRY(check_array(dK, (int64_t)p->B * (p->H / groups(p)) * N * p->d));
    HILS_TRY(check_array(dLQ, (int64_t)p->B * p->H * C * p->d));
    BwdSummarizeArgs a;
    a.K = {K.ptr, K.sb, K.sh, K.st};
    a.LQ = {LQ.ptr, LQ.sb, LQ.sh, LQ.st};
    a.dKsum = dKsum;
    a.dBsum = dBsum;
    a.dK = dK;
    a.dLQ = dLQ;
    a.B = p->B;
    a.H = p->H;
    a.N = N;
    a.C = C;
    a.G = groups(p);
    a.scale = scale;
    return launch_summarize_backward(p->dtype, p->d, a, stream);
}

int hils_select(const hils_params *p, hils_ctensor Qcal, int Lq, const int32_t *qpos, hils_ctensor Ksum,
                const float *Bsum, int C, int32_t *idx, float *score, int32_t *nsel, void *workspace,
                size_t ws_bytes, cudaStream_t stream) {
    SelectArgs a{};
    int64_t nq = 0;
    HILS_TRY(prepare_select(p, Qcal, Lq, qpos, 0, Ksum, Bsum, C, idx, score, nsel, &a, &nq));
    if (nq == 0) return HILS_OK;
    HILS_TRY(check_workspace(workspace, ws_bytes, select_ws_bytes((int)nq, C, a.path)));
    a.ws = workspace;
    return launch_select(p->dtype, p->d, a, stream);
}

int hils_attend_prefill(const hils_params *p, hils_ctensor Q, hils_ctensor K, hils_ctensor V, int N,
                        const int32_t *idx, const float *score, const int32_t *nsel, hils_tensor O, float *lse,
                        void *workspace, size_t ws_bytes, cudaStream_t stream) {
    float scale;
    HILS_TRY(check_params(p, &scale));
    if (N < 0) return HILS_ERR_INVALID_ARG;
    const int64_t nq = (int64_t)p->B * p->H * N;
    HILS_TRY(check_view(Q.ptr, Q.sb, Q.sh, Q.st, N, p));
    HILS_TRY(check_view(K.ptr, K.sb, K.sh, K.st, N, p));
    HILS_TRY(check_view(V.ptr, V.sb, V.sh, V.st, N, p));
    HILS_TRY(check_view(O.ptr, O.sb, O.sh, O.st, N, p));
    HILS_TRY(check_array(idx, nq / groups(p) * p->K));
    HILS_TRY(check_array(score, nq * p->K));
    HILS_TRY(check_array(nsel, p->K > 0 ? nq / groups(p) : 0));
    HILS_TRY(check_array(lse, 0));
    HILS_TRY(check_workspace(workspace, ws_bytes, kPrefillWsBytes));
    if (nq == 0) return HILS_OK;
    AttendArgs a{};
    a.Q = {Q.ptr, Q.sb, Q.sh, Q.st};
    a.K = {K.ptr, K.sb, K.sh, K.st};
    a.V = {V.ptr, V.sb, V.sh, V.st};
    a.O = {O.ptr, O.sb, O.sh, O.st};
    a.lse = lse;
    a.idx = idx;
    a.score = score;
    a.nsel = nsel;
    a.qpos = nullptr;
    a.cache_len = nullptr;
    a.B = p->B;
    a.H = p->H;
    a.Lq = N;
    a.topk = p->K;
    a.W = p->W;
    a.scale = scale;
    a.units = decode_units(p);
    a.ws = workspace;
    a.G = groups(p);
    a.wait_ns = work_wait_ns(p->flags);
    if (attend_prefill_tc_supported(p->dtype, p->d, N))
        return launch_attend_prefill_tc(a, N, static_cast<uint32_t *>(workspace), stream);
    return launch_attend_prefill_general(p->dtype, p->d, a, stream);
}

int hils_attend_decode(const hils_params *p, hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc,
                       const int32_t *cache_len, const int32_t *idx, const float *score, const int32_t *nsel,
                       hils_tensor O, float *lse, void *workspace, size_t ws_bytes, cudaStream_t stream) {
    AttendArgs a{};
    HILS_TRY(prepare_attend_decode(p, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse, &a));
    const int64_t nq = (int64_t)p->B * p->H;
    if (nq == 0) return HILS_OK;
    HILS_TRY(check_workspace(workspace, ws_bytes, attend_decode_ws_bytes((int)nq, a.units, p->d)));
    a.ws = workspace;
    return launch_attend_decode(p->dtype, p->d, a, stream);
}

int hils_decode(const hils_params *p, hils_ctensor Qcal, hils_ctensor Ksum, const float *Bsum, int C,
                hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc, const int32_t *cache_len, int32_t *idx,
                float *score, int32_t *nsel, hils_tensor O, float *lse, void *workspace, size_t ws_bytes,
                cudaStream_t stream) {
    SelectArgs sa{};
    int64_t nq = 0;
    HILS_TRY(prepare_select(p, Qcal, 1, cache_len, -1, Ksum, Bsum, C, idx, score, nsel, &sa, &nq));
    AttendArgs aa{};
    HILS_TRY(prepare_attend_decode(p, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse, &aa));
    if (nq == 0) return HILS_OK;
    const size_t sel_bytes = decode_select_part(select_ws_bytes((int)nq, C, sa.path));
    HILS_TRY(check_workspace(workspace, ws_bytes, sel_bytes + attend_decode_ws_bytes((int)nq, aa.units, p->d)));
    sa.ws = workspace;
    aa.ws = static_cast<uint8_t *>(workspace) + sel_bytes;
    // the select's first kernel waits for every earlier write on the stream before it
    // reads anything, and each later kernel of the chain is scheduled only after the one
    // before it passed that point: the attend's window tiles need not wait for the select
    aa.window_early = 1;
    HILS_TRY(launch_select(p->dtype, p->d, sa, stream));
    return launch_attend_decode(p->dtype, p->d, aa, stream);
}

}  // extern "C"
