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
// An FP32 evaluation is accepted unless it lies within a margin of a bf16
// rounding midpoint (where its own error could move it across), or near the
// FP32 subnormal range; those cases are recomputed in double.  The margins
// bound the FP32 evaluation's error on each range, in FP32 ulps of the
// result:
//   y >= 10        : y itself (1 - Phi(y) < 8e-24, far below half a bf16 ulp).
//   0 <= y < 10    : 0.5 y erfcf(-y / sqrt 2): erfcf's few ulps and two
//                    roundings; erfc(-t) in [1, 2] barely amplifies the
//                    argument's rounding.  Margin 32 ulps.
//   -3.125 <= y < 0: the same formula; erfc(t) amplifies the argument's
//                    relative rounding (~2^-23.4) by up to 2 t^2 < 10.
//                    Margin 32 ulps.
//   -10 <= y < -3.125: the same, amplification up to 2 t^2 = 100.  Margin
//                    128 ulps.
//   y < -10        : with x = -y, Phi(y) = phi(x) / x (1 - 1/x^2 + 3/x^4 -
//                    15/x^6 + 105/x^8 - ...), an alternating asymptotic
//                    series whose first omitted term bounds the error (945 /
//                    x^10 < 2^-23.3); so GELU(y) = -phi(x) S(1/x^2) with
//                    phi(x) = exp(-x^2/2) / sqrt(2 pi), x^2 exact in FP32.
//                    Margin 64 ulps; results below 2^-120 (x > ~12.9, bf16
//                    subnormals and underflow) go to double.
// In double, the value is rounded to bf16 from its exact binary value.  A
// double result exactly on a midpoint arises only for subnormal y, where it
// is y / 2 with the y^2 / sqrt(2 pi) term rounded away; the true value lies
// above it (GELU(y) - y / 2 = y (Phi(y) - 1/2) > 0), so such a tie rounds up.
// Every bf16 input is checked against a 50-digit reference through the
// library's tests.
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
    float h;
    uint32_t margin;
    if (y >= -10.0f) {
        h = __fmul_rn(__fmul_rn(0.5f, y), erfcf(__fmul_rn(-y, 0.70710678118654752f)));
        margin = y >= -3.125f ? 32u : 128u;
    } else {
        const float x2 = __fmul_rn(y, y);  // exact: y has 8 significant bits
        const float u = __frcp_rn(x2);
        const float s = __fmaf_rn(-u, __fmaf_rn(-3.0f * u, __fmaf_rn(-5.0f * u, __fmaf_rn(-7.0f, u, 1.0f), 1.0f), 1.0f),
                                  1.0f);
        h = -__fmul_rn(__fmul_rn(expf(-0.5f * x2), 0.39894228040143268f), s);
        margin = 64u;
    }
    const uint32_t hb = __float_as_uint(h);
    const uint32_t low = hb & 0xFFFFu;
    if ((hb & 0x7F800000u) < (7u << 23) || (low > 0x8000u - margin && low < 0x8000u + margin))
        return gelu_bf16_slow(y);
    return (hb + 0x7FFFu + ((hb >> 16) & 1u)) >> 16;
}

// ---------------------------------------------------------------- table form
// The kernels that apply GELU to many values read the results for the 4096
// bf16 inputs with 2^-12 <= |y| < 2^4 (16 exponents x 128 mantissas x 2
// signs: all but a sliver of any activation) from an 8 KB shared-memory
// table, filled once per CTA by gelu_bf16 above (FP32, double near a
// rounding midpoint: correctly rounded either way).  Outside it:
//   |y| >= 16      : y for y > 0; -0 for y < 0 (|GELU(y)| < 2^-134, below
//                    half the smallest bf16 subnormal).
//   y = +-0        : y.
//   |y| < 2^-12    : GELU(y) = y/2 + phi(0) y^2 (1 - y^2/6) + O(y^6), the
//                    Taylor series of y Phi(y) at 0; the omitted terms are
//                    far below 2^-25 of the value, FP32 evaluation adds a few
//                    ulps: margin 16 ulps, else (and for subnormal inputs or
//                    FP32-subnormal results) the double path.
// Table entry s << 11 | (e - 115) << 7 | m holds GELU of the bf16 with sign
// s, biased exponent e (115..130) and mantissa m.
constexpr int kGeluTab = 4096;

__device__ __forceinline__ void gelu_table_build(uint16_t* tab, int tid, int nthreads) {
    for (int i = tid; i < kGeluTab; i += nthreads) {
        const uint32_t b = ((uint32_t)(i >> 11) << 15) | ((115u + ((uint32_t)i >> 7 & 15u)) << 7) | ((uint32_t)i & 127u);
        tab[i] = (uint16_t)gelu_bf16(b);
    }
}

// One value (low 16 bits of ybits) by the table and the cases around it.
__device__ __forceinline__ uint32_t gelu_bf16_tab(uint32_t ybits, const uint16_t* tab) {
    ybits &= 0xFFFFu;
    const uint32_t e = (ybits >> 7) & 0xFFu;
    if (e - 115u <= 15u) return tab[((ybits >> 4) & 0x800u) | ((e - 115u) << 7) | (ybits & 0x7Fu)];
    if (e > 130u) return (ybits & 0x8000u) ? 0x8000u : ybits;
    if ((ybits & 0x7FFFu) == 0u) return ybits;
    if (e == 0u) return gelu_bf16_slow(__uint_as_float(ybits << 16));
    const float y = __uint_as_float(ybits << 16);
    const float y2 = __fmul_rn(y, y);
    const float c = __fmaf_rn(y2, -0.066490380066905446f, 0.39894228040143268f);  // phi(0) (1 - y^2 / 6)
    const float h = __fmul_rn(__fmaf_rn(c, y, 0.5f), y);
    const uint32_t hb = __float_as_uint(h);
    const uint32_t low = hb & 0xFFFFu;
    if ((hb & 0x7F800000u) < (7u << 23) || (low > 0x8000u - 16u && low < 0x8000u + 16u))
        return gelu_bf16_slow(y);
    return (hb + 0x7FFFu + ((hb >> 16) & 1u)) >> 16;
}

// Both halves of a word, one at a time: the rare case of the packed form,
// kept out of line so that the common path stays short.
__device__ __noinline__ uint32_t gelu_bf16x2_rare(uint32_t w, const uint16_t* tab) {
    return gelu_bf16_tab(w, tab) | (gelu_bf16_tab(w >> 16, tab) << 16);
}

// Two bf16 values packed in a word (element 0 in the low half).  Both
// exponents are offset by 141 in their own 16-bit lanes (no carry between
// them: 255 + 141 < 2^16), so each lies in [256, 272) exactly when its value
// is inside the table, and both table indices are assembled in one word.
// The indices are in range whatever the exponents; the loads go first and
// the rare case replaces their result.
__device__ __forceinline__ uint32_t gelu_bf16x2_tab(uint32_t w, const uint16_t* tab) {
    const uint32_t v = ((w >> 7) & 0x00FF00FFu) + 0x008D008Du;
    const uint32_t i = ((w >> 4) & 0x08000800u) | ((v & 0x000F000Fu) << 7) | (w & 0x007F007Fu);
    uint32_t r = (uint32_t)tab[i & 0xFFFFu] | ((uint32_t)tab[i >> 16] << 16);
    if ((v & 0xFFF0FFF0u) != 0x01000100u) r = gelu_bf16x2_rare(w, tab);
    return r;
}

}  // namespace ft
