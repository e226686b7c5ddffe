// hils_selftest_fast_math: evaluates the library's FMA-pipe helpers (fast_math.cuh) on
// caller-given inputs, so that their error bounds can be checked against float64
// references outside the kernels that use them.
#include "fast_math.cuh"
#include "hils_internal.cuh"

namespace hils {
namespace {

__global__ void fast_math_kernel(const float *x, const float *z, int n, float *exp2_out, float *recip_out) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        exp2_out[i] = exp2_fma(x[i]);
        recip_out[i] = recip_newton(z[i]);
    }
}

}  // namespace
}  // namespace hils

extern "C" int hils_selftest_fast_math(const float *x, const float *z, int n, float *exp2_out, float *recip_out,
                                       cudaStream_t stream) {
    using namespace hils;
    if (n < 0) return HILS_ERR_INVALID_ARG;
    if (n == 0) return HILS_OK;
    if (!x || !z || !exp2_out || !recip_out) return HILS_ERR_INVALID_ARG;
    const int blocks = (int)(((int64_t)n + 255) / 256 < 4096 ? ((int64_t)n + 255) / 256 : 4096);
    fast_math_kernel<<<blocks, 256, 0, stream>>>(x, z, n, exp2_out, recip_out);
    return record_cuda_error(cudaGetLastError());
}
