// hils_attend_decode_noalloc: the decode attend with its scratch memory compiled into
// the library, for callers that cannot allocate device memory themselves.
//
// The scratch is one fixed array in device global memory. Every GPU that loads this
// library holds it until the process exits. On the host its name is only a stand-in
// symbol, not a device address, so the address is looked up with
// cudaGetSymbolAddress once per device (with that device current) and handed to the
// kernels as an ordinary workspace pointer.
#include "hils_internal.cuh"

namespace hils {
namespace {

// Capacity of the built-in scratch: (B*H) x units x (d+1) floats plus one arrival
// counter per (b, h) must fit. 512K decode (B1 H32, K16, W512) needs about 0.4 MiB,
// the B=8 128K workload about 3.2 MiB.
constexpr size_t kScratchBytes = size_t(4) << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

struct ScratchCache {
    void *addr[64] = {};
    unsigned long long ready = 0;  // bit per device ordinal
};
ScratchCache g_cache;

hils_status scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return record_cuda_error(e);
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (__atomic_load_n(&g_cache.ready, __ATOMIC_ACQUIRE) & bit)) {
        *out = g_cache.addr[dev];
        return HILS_OK;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return record_cuda_error(e);
    if (bit) {
        g_cache.addr[dev] = p;
        __atomic_fetch_or(&g_cache.ready, bit, __ATOMIC_RELEASE);
    }
    *out = p;
    return HILS_OK;
}

}  // namespace
}  // namespace hils

extern "C" int hils_attend_decode_noalloc(const hils_params *p, hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc,
                                          const int32_t *cache_len, const int32_t *idx, const float *score,
                                          const int32_t *nsel, hils_tensor O, float *lse, cudaStream_t stream) {
    using namespace hils;
    // every argument check runs before anything touches the shared scratch, so a call
    // that is rejected leaves no work queued on the stream
    const int chk = check_attend_decode_args(p, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse);
    if (chk != HILS_OK) return chk;
    const size_t need = hils_workspace_bytes(p, HILS_CALL_ATTEND_DECODE, 1, 0);
    if (need > kScratchBytes) return HILS_ERR_WORKSPACE;  // beyond the built-in capacity
    void *scratch = nullptr;
    if (need > 0) {
        const hils_status st = scratch_address(&scratch);
        if (st != HILS_OK) return st;
        // the arrival counters and flags at the front of the scratch must start at zero
        const size_t counters = attend_decode_counter_bytes(p->B * p->H);
        const hils_status mz = record_cuda_error(cudaMemsetAsync(scratch, 0, counters, stream));
        if (mz != HILS_OK) return mz;
    }
    return hils_attend_decode(p, Q, Kc, Vc, cache_len, idx, score, nsel, O, lse, scratch, kScratchBytes, stream);
}
