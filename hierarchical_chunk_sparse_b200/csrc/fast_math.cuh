// Scalar helpers on the FMA pipe, for kernels whose MUFU unit is busy with the softmax
// exponentials: a reciprocal and a base-2 exponential. Both are this library's own
// (a numerically fitted seed with Newton steps; a fitted polynomial), checked on the
// GPU against float64 references by hils_selftest_fast_math.
#pragma once
#include <cuda_runtime.h>

namespace hils {

// 1/z for a normal positive z on the FMA pipe: an integer-subtraction seed (relative
// error at most 5.1e-2, constant fitted numerically over one binade) and two Newton
// steps r <- r (2 - z r), which square the error: below 7e-6 plus rounding.
__device__ __forceinline__ float recip_newton(float z) {
    float r = __int_as_float(0x7ef311c2 - __float_as_int(z));
    r = fmaf(r, fmaf(-z, r, 1.f), r);
    r = fmaf(r, fmaf(-z, r, 1.f), r);
    return r;
}

// 2^x on the FMA pipe (no MUFU), for finite x: x = j + f with j = round(x) (the
// 1.5 * 2^23 shifter) and f in [-1/2, 1/2]; 2^f by a degree-5 polynomial fitted here for
// relative error (iteratively reweighted least squares on Chebyshev nodes; at most
// 2.4e-7 in float32 Horner form); 2^j added to the exponent field. x is clamped to
// [-125, 127] so the result stays a normal float (2^-125 stands for anything smaller).
__device__ __forceinline__ float exp2_fma(float x) {
    x = fminf(fmaxf(x, -125.f), 127.f);
    const float t = x + 12582912.f;
    const float f = x - (t - 12582912.f);
    float p = 1.327647129e-03f;
    p = fmaf(p, f, 9.675540961e-03f);
    p = fmaf(p, f, 5.550713092e-02f);
    p = fmaf(p, f, 2.402212024e-01f);
    p = fmaf(p, f, 6.931469440e-01f);
    p = fmaf(p, f, 1.000000119e+00f);
    return __int_as_float(__float_as_int(p) + ((__float_as_int(t) - 0x4b400000) << 23));
}

}  // namespace hils
