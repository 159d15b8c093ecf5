// ft_gelu.cuh -- the activation between a DiT block's MLP linears, GELU,
// on bf16 values, rounded once to bf16 (round to nearest even): the
// function the fused MLP applies to the FC1 output before quantizing it for
// FC2 (FourTune page, section 3.3, "MLP Fusion").
//
//   GELU(y) = y Phi(y) = 0.5 y erfc(-y / sqrt 2)
//
// The erfc form keeps its relative accuracy in the tail (1 + erf(t) would
// cancel for y << 0).  A bf16 input takes one of 65536 values; the result
// must be the correctly rounded bf16 of the exact GELU for every one of them.
//   y >= 10        : y itself (1 - Phi(y) < 8e-24, far below half a bf16 ulp
//                    of y).
//   -10 <= y < 10  : FP32 first.  The FP32 evaluation's relative error is
//                    below 2^-16 (erfcf's few ulps plus the argument's
//                    rounding amplified by erfc's slope, 2 t^2 2^-23 at
//                    t = 7.07); unless the FP32 value lies within 256 FP32
//                    ulps (2^-15 relative) of a bf16 rounding midpoint, its
//                    RNE rounding to bf16 is the correct one.
//   otherwise      : double, rounded to bf16 from its exact binary value;
//                    that covers the midpoint neighbourhoods, y < -10 and
//                    results near or below the FP32 normal range (bf16
//                    subnormals).  A double result exactly on a midpoint
//                    arises only for subnormal y, where it is y / 2 with the
//                    y^2 / sqrt(2 pi) term rounded away; the true value lies
//                    above it (GELU(y) - y / 2 = y (Phi(y) - 1/2) > 0), so such
//                    a tie rounds up.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ft {

// bf16 bits of the double h, rounded to nearest (ties toward +infinity, the
// side the exact GELU lies on whenever its double value is a tie).
__device__ __noinline__ uint32_t gelu_bf16_from_double(double h) {
    if (h == 0.0) return __double_as_longlong(h) < 0 ? 0x8000u : 0u;
    const double a = fabs(h);
    const int e = ilogb(a);
    const int qe = max(e - 7, -133);      // bf16 quantum at a: 8 significant bits, subnormals below 2^-126
    const double m = ldexp(a, -qe);       // exact (a power-of-two scaling)
    double r = floor(m);
    const double frac = m - r;
    if (frac > 0.5 || (frac == 0.5 && h > 0.0)) r += 1.0;
    const float v = (float)ldexp(h > 0.0 ? r : -r, qe);  // exact: at most 9 significant bits
    return __float_as_uint(v) >> 16;
}

__device__ __noinline__ uint32_t gelu_bf16_slow(float y) {
    const double yd = (double)y;
    return gelu_bf16_from_double(0.5 * yd * erfc(-yd * 0.70710678118654752440));
}

// GELU of one bf16 value (low 16 bits of ybits), as bf16 bits.
__device__ __forceinline__ uint32_t gelu_bf16(uint32_t ybits) {
    ybits &= 0xFFFFu;
    const float y = __uint_as_float(ybits << 16);
    if (!(y < 10.0f)) return ybits;  // y >= 10 (and +inf); NaN is outside the contract
    if (y < -10.0f) return gelu_bf16_slow(y);
    const float h = __fmul_rn(__fmul_rn(0.5f, y), erfcf(__fmul_rn(-y, 0.70710678118654752f)));
    const uint32_t hb = __float_as_uint(h);
    const uint32_t low = hb & 0xFFFFu;
    if ((hb & 0x7F800000u) < (7u << 23) || (low > 0x8000u - 256u && low < 0x8000u + 256u))
        return gelu_bf16_slow(y);
    return (hb + 0x7FFFu + ((hb >> 16) & 1u)) >> 16;
}

// GELU of two bf16 values packed in a word (element 0 in the low half).
__device__ __forceinline__ uint32_t gelu_bf16x2(uint32_t w) {
    return gelu_bf16(w) | (gelu_bf16(w >> 16) << 16);
}

}  // namespace ft
