// rope_angle.cuh -- rotation angle phi = m * theta'_i for large positions.
//
// The fp32 product m * theta loses up to 2^-7 rad at m ~ 1.3e5, so the angle
// is formed in fp64 (exact for |m| < 2^29: 29 + 24 bits <= 53), reduced to
// [-pi, pi] by subtracting the nearest multiple of 2 pi (a two-part
// Cody-Waite constant, 2 pi = hi + lo), and only then rounded to fp32.
#pragma once
#include <cuda_runtime.h>

namespace lcx {

// 2 pi split into the fp64 value nearest to it and the remainder.
constexpr double kTwoPiHi = 6.283185307179586;
constexpr double kTwoPiLo = 2.4492935982947064e-16;
constexpr double kInvTwoPi = 0.15915494309189535;

// m * theta reduced to [-pi, pi] (fp32).
__device__ __forceinline__ float rope_reduced_angle(long long m, float theta) {
    const double phi = static_cast<double>(m) * static_cast<double>(theta);
    const double k = rint(phi * kInvTwoPi);
    double r = fma(-k, kTwoPiHi, phi);
    r = fma(-k, kTwoPiLo, r);
    return static_cast<float>(r);
}

// Accurate (libm) cosine and sine of m * theta.
__device__ __forceinline__ void rope_sincos(long long m, float theta, float *c, float *s) {
    sincosf(rope_reduced_angle(m, theta), s, c);
}

// Fast (hardware approximation) cosine and sine of m * theta; absolute error
// about 2^-21 on the reduced argument -- ample for bf16 operands.
__device__ __forceinline__ void rope_sincos_fast(long long m, float theta, float *c, float *s) {
    __sincosf(rope_reduced_angle(m, theta), s, c);
}

}  // namespace lcx
