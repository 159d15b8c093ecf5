// ft_nvfp4.cuh -- the NVFP4 block encoder used by every quantizing kernel.
//
// Encoding (FourTune page, section 3.2 block quantization; the page names
// NVFP4, whose elements are E2M1 with one E4M3 scale per block and an FP32
// tensor scale):
//   g   = amax_tensor / 2688              (1 when amax_tensor == 0)
//   sd  = E4M3_rne_satfinite(amax_block / (6 g))
//   q   = x / (sd g)                      (IEEE single, round to nearest even)
//   code= E2M1_rne_satfinite(q), sign of x kept; 0 when sd == 0
// Every FP32 step is an explicitly rounded intrinsic (no contraction), so the
// codes and scales are bit-identical to a scalar IEEE implementation.
#pragma once

#include "ft_ptx.cuh"

namespace ft {

// Byte offset of the scale of (row r, 16-column block b) in the slab layout
// the FP4 GEMM copies into tensor memory: [ceil(rows/128)][cols/64][512],
// byte 16 l + 4 i + (b % 4) of slab (r / 128, b / 4) with r % 128 = 32 i + l.
__host__ __device__ __forceinline__ int64_t slab_offset(int64_t r, int64_t b, int64_t cols) {
    return ((r >> 7) * (cols >> 6) + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

struct QTensor {
    float g;      // decode tensor scale
    float six_g;  // RN(6 g)
};

__device__ __forceinline__ QTensor make_qtensor(float amax) {
    QTensor t;
    t.g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
    t.six_g = __fmul_rn(6.0f, t.g);
    return t;
}

// RN(v) to E4M3 with saturation to 448; returns the byte.
__device__ __forceinline__ uint32_t e4m3_encode(float v) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
    return out & 0xFFu;
}

// Exact value of an E4M3 byte.
__device__ __forceinline__ float e4m3_decode(uint32_t b) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)b));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Eight non-negative values -> eight E2M1 magnitude codes (RNE, saturating
// to 6), value i in nibble i.  In cvt...e2m1x2 the second source lands in the
// low nibble.
__device__ __forceinline__ uint32_t e2m1x8_encode(const float (&a)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]),
          "f"(a[7]));
    return out;
}

// RN(x / d) for d a normal float in [2^-60, 2^60] and x non-negative:
// y = RN(1/d) is within half an ulp of 1/d and q0 = RN(x y) is faithful, so
// one correction step with the exact remainder x - q0 d (an FMA) returns the
// correctly rounded quotient (Markstein's theorem; see Muller et al.,
// "Handbook of Floating-Point Arithmetic", division by Newton-Raphson).  The
// range limit keeps the remainder clear of the subnormal range whenever the
// quotient is large enough to matter for E2M1 (>= 2^-3).
__device__ __forceinline__ float div_by_recip(float x, float d, float y) {
    float q = __fmul_rn(x, y);
    float r = __fmaf_rn(-q, d, x);
    return __fmaf_rn(r, y, q);
}

// bf16 bit pattern (low 16 bits of w) -> |value| as float
__device__ __forceinline__ float bf16_lo_abs(uint32_t w) { return __uint_as_float((w & 0x7FFFu) << 16); }
__device__ __forceinline__ float bf16_hi_abs(uint32_t w) { return __uint_as_float(w & 0x7FFF0000u); }

// Max of |x| over 8 packed bf16 pairs, as the bf16 magnitude bits << 16.
__device__ __forceinline__ uint32_t amax_bits_16(const uint32_t (&w)[8]) {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
    m = max(m & 0xFFFFu, m >> 16);
    return m << 16;
}

// Sign bits of 8 bf16 values (w[0..3]) placed at bit 3 of each nibble.
__device__ __forceinline__ uint32_t sign_nibbles_8(uint32_t w0, uint32_t w1, uint32_t w2,
                                                   uint32_t w3) {
    uint32_t s = 0;
    s |= (w0 >> 15) & 1u;
    s |= ((w0 >> 31) & 1u) << 4;
    s |= ((w1 >> 15) & 1u) << 8;
    s |= ((w1 >> 31) & 1u) << 12;
    s |= ((w2 >> 15) & 1u) << 16;
    s |= ((w2 >> 31) & 1u) << 20;
    s |= ((w3 >> 15) & 1u) << 24;
    s |= ((w3 >> 31) & 1u) << 28;
    return s << 3;
}

// Codes of 8 elements (w0..w3 = 4 bf16 pairs) for divisor d, as 8 nibbles.
__device__ __forceinline__ uint32_t encode8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                            float d, float y, bool fast) {
    float a[8] = {bf16_lo_abs(w0), bf16_hi_abs(w0), bf16_lo_abs(w1), bf16_hi_abs(w1),
                  bf16_lo_abs(w2), bf16_hi_abs(w2), bf16_lo_abs(w3), bf16_hi_abs(w3)};
    float q[8];
    if (fast) {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = div_by_recip(a[i], d, y);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(a[i], d);
    }
    return e2m1x8_encode(q) | sign_nibbles_8(w0, w1, w2, w3);
}

// Per-block divisor setup.  Returns false when the block is all zero scale
// (sd == 0: every code is 0).
struct BlockDiv {
    float d, y;
    bool fast;
};

__device__ __forceinline__ bool block_divisor(float amax_b, const QTensor& t, uint32_t& sbyte,
                                              BlockDiv& bd) {
    float sf = __fdiv_rn(amax_b, t.six_g);
    sbyte = e4m3_encode(sf);
    float sd = e4m3_decode(sbyte);
    if (sd == 0.0f) return false;
    bd.d = __fmul_rn(sd, t.g);
    bd.fast = (bd.d >= 0x1p-60f) && (bd.d <= 0x1p60f);
    bd.y = bd.fast ? __frcp_rn(bd.d) : 0.0f;
    return true;
}

// Quantize one 1x16 block held as 8 bf16 pairs.  Returns 16 codes packed in
// 8 bytes (element 0 in the low nibble of byte 0) and the scale byte.
__device__ __forceinline__ uint2 quant_block16(const uint32_t (&w)[8], const QTensor& t,
                                               uint32_t& sbyte) {
    float amax_b = __uint_as_float(amax_bits_16(w));
    BlockDiv bd;
    if (!block_divisor(amax_b, t, sbyte, bd)) return make_uint2(0u, 0u);
    uint2 r;
    r.x = encode8(w[0], w[1], w[2], w[3], bd.d, bd.y, bd.fast);
    r.y = encode8(w[4], w[5], w[6], w[7], bd.d, bd.y, bd.fast);
    return r;
}


// ------------------------------------------------------------------------
// Throughput path.  The divisor d = RN(sd g) of a block depends only on its
// scale byte, so each CTA tabulates d and y = RN(1/d) for the 126 positive
// finite E4M3 values once (QTable, in shared memory); per element the exact
// quotient then costs one packed multiply and two packed FMAs on f32x2
// pairs.  The sign of x is ORed back after the division (the correction step
// turns -0 / d into +0), and cvt...e2m1x2 encodes sign and magnitude.
// Bit-identical to quant_block16 (same IEEE definition).

struct QTable {
    float d[128];
    float y[128];  // 0 marks a divisor outside [2^-60, 2^60]: use IEEE division
};

struct QTensorFast {
    float g, six_g, y6;  // y6 = RN(1/six_g), 0 when six_g is outside the safe range
};

__device__ __forceinline__ QTensorFast make_qtensor_fast(float amax) {
    QTensor t = make_qtensor(amax);
    QTensorFast f;
    f.g = t.g;
    f.six_g = t.six_g;
    f.y6 = (t.six_g >= 0x1p-60f && t.six_g <= 0x1p60f) ? __frcp_rn(t.six_g) : 0.0f;
    return f;
}

// Fill the table cooperatively (threads tid of nthreads).  Call before a
// barrier that precedes the first lookup.
__device__ __forceinline__ void build_qtable(QTable& tab, float g, int tid, int nthreads) {
    for (int s = tid; s < 128; s += nthreads) {
        float d = 0.0f, y = 0.0f;
        if (s >= 1 && s <= 0x7E) {
            d = __fmul_rn(e4m3_decode((uint32_t)s), g);
            y = (d >= 0x1p-60f && d <= 0x1p60f) ? __frcp_rn(d) : 0.0f;
        }
        tab.d[s] = d;
        tab.y[s] = y;
    }
}

__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Scale byte of a block from its amax (Markstein quotient when y6 != 0).
__device__ __forceinline__ uint32_t scale_byte_fast(float amax_b, const QTensorFast& t) {
    float sf;
    const float q = __fmul_rn(amax_b, t.y6);
    if (t.y6 != 0.0f && q < 0x1p100f) {
        const float r = __fmaf_rn(-q, t.six_g, amax_b);
        sf = __fmaf_rn(r, t.y6, q);
    } else {
        // no reciprocal, or a quotient far beyond the E4M3 range (a caller
        // amax below the true one): IEEE division, which saturates cleanly
        sf = __fdiv_rn(amax_b, t.six_g);
    }
    return e4m3_encode(sf);
}

// Codes of 8 elements (4 bf16 pairs) given the block divisor d and y.
__device__ __forceinline__ uint32_t encode8_fast(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                                 float d, float y) {
    const uint32_t w[4] = {w0, w1, w2, w3};
    const uint64_t Y = f2pack(y, y);
    const uint64_t ND = f2pack(-d, -d);
    uint32_t out;
    float q[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = w[i] << 16, hi = w[i] & 0xFFFF0000u;
        const uint64_t X = f2pack(__uint_as_float(lo), __uint_as_float(hi));
        uint64_t Q = mul_f32x2(X, Y);
        const uint64_t R = fma_f32x2(Q, ND, X);
        Q = fma_f32x2(R, Y, Q);
        float qa, qb;
        f2unpack(Q, qa, qb);
        q[2 * i] = __uint_as_float(__float_as_uint(qa) | (lo & 0x80000000u));
        q[2 * i + 1] = __uint_as_float(__float_as_uint(qb) | (hi & 0x80000000u));
    }
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return out;
}

// One 1x16 block through the table, its max|x| given as float bits
// (amax_bits_16 of the same block).  Returns the 8 code bytes; *sbyte the
// scale.
__device__ __forceinline__ uint2 quant_block16_fast_m(const uint32_t (&w)[8], uint32_t amax_bits,
                                                      const QTensorFast& t, const QTable& tab,
                                                      uint32_t& sbyte) {
    const float amax_b = __uint_as_float(amax_bits);
    sbyte = scale_byte_fast(amax_b, t);
    const float d = tab.d[sbyte];
    const float y = tab.y[sbyte];
    uint2 r;
    if (sbyte == 0) {
        r = make_uint2(0u, 0u);
    } else if (y != 0.0f && sbyte != 0x7Eu) {
        // below the top scale every quotient stays under ~13, so x * y cannot
        // overflow; the saturated top scale (a tensor's largest block, or a
        // caller amax below the true one) takes the IEEE path
        r.x = encode8_fast(w[0], w[1], w[2], w[3], d, y);
        r.y = encode8_fast(w[4], w[5], w[6], w[7], d, y);
    } else {
        r.x = encode8(w[0], w[1], w[2], w[3], d, 0.0f, false);
        r.y = encode8(w[4], w[5], w[6], w[7], d, 0.0f, false);
    }
    return r;
}

// One 1x16 block through the table.  Returns the 8 code bytes; *sbyte the scale.
__device__ __forceinline__ uint2 quant_block16_fast(const uint32_t (&w)[8], const QTensorFast& t,
                                                    const QTable& tab, uint32_t& sbyte) {
    return quant_block16_fast_m(w, amax_bits_16(w), t, tab, sbyte);
}


// ------------------------------------------------------------------------
// Multiply path.  For most divisors d the product RN(x * y), y = RN(1/d),
// already encodes every bf16 x exactly like the correctly rounded RN(x / d):
// the two differ by at most an ulp of FP32, which changes the E2M1 code only
// for an x within that ulp of one of the seven rounding boundaries
// {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5} * d.  Both encodings are monotone
// step functions of |x|, so they agree on every bf16 value when they agree on
// the few bf16 values around each boundary; QTableM checks exactly those
// once per scale byte.  When RN(1/d) fails, its two FP32 neighbours are
// tried: they move the product by one more ulp at most, far less than the
// spacing of bf16 values, so the same few candidates still decide.  ym[]
// keeps the first multiplier that passes (0: none does, IEEE division).
// The multiply also carries the sign (a -0 input gives -0 and code 0x8), so
// an element costs half a packed multiply and half a conversion.
// Bit-identical to quant_block16 (same IEEE definition).

constexpr int QT_NY = 3;  // multipliers tried: RN(1/d), then one ulp below and above

struct QTableM {
    float d[128];
    float y[128];           // 0: divisor outside [2^-60, 2^60] (IEEE division)
    float ym[128];          // the multiplier that is exact for every bf16 x, else 0
    uint32_t bad[QT_NY][4]; // scratch of the check: one bit per (multiplier, scale byte)
};

__device__ __forceinline__ uint32_t e2m1_encode1(float q) {
    uint16_t out;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
        "cvt.u16.u8 %0, b;\n\t}"
        : "=h"(out)
        : "f"(0.0f), "f"(q));
    return out & 0xFu;
}

// Candidate multiplier j of a positive normal y: y, y - 1 ulp, y + 1 ulp.
__device__ __forceinline__ float qt_multiplier(float y, int j) {
    const uint32_t u = __float_as_uint(y);
    return __uint_as_float(j == 0 ? u : (j == 1 ? u - 1u : u + 1u));
}

// Step 1 of 3 (a barrier between steps): divisors and reciprocals.
__device__ __forceinline__ void build_qtable_m1(QTableM& tab, float g, int tid, int nthreads) {
    for (int s = tid; s < 128; s += nthreads) {
        float d = 0.0f, y = 0.0f;
        if (s >= 1 && s <= 0x7E) {
            d = __fmul_rn(e4m3_decode((uint32_t)s), g);
            y = (d >= 0x1p-60f && d <= 0x1p60f) ? __frcp_rn(d) : 0.0f;
        }
        tab.d[s] = d;
        tab.y[s] = y;
    }
    if (tid < QT_NY * 4) (&tab.bad[0][0])[tid] = 0u;
}

// Step 2: the exactness check of the multiply path, for each candidate
// multiplier, four threads per scale byte (boundaries k = part, part + 4).
__device__ __forceinline__ void build_qtable_m2(QTableM& tab, int tid, int nthreads) {
    for (int i = tid; i < QT_NY * 512; i += nthreads) {
        const int j = i >> 9, s = i & 127, part = (i >> 7) & 3;
        const float d = tab.d[s], y = tab.y[s];
        if (s == 0 || s >= 0x7E || y == 0.0f) continue;  // these never take the multiply path
        const float yj = qt_multiplier(y, j);
        bool ok = true;
        for (int k = part; k < 7; k += 4) {
            // rounding boundary k of the E2M1 grid: 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5
            const float bk = k < 4 ? 0.25f + 0.5f * (float)k : (k == 4 ? 2.5f : (k == 5 ? 3.5f : 5.0f));
            // x0: the largest bf16 value <= bk d (RZ keeps the product at or
            // below the exact one, truncation then keeps a bf16 value below it)
            const uint32_t x0 = __float_as_uint(__fmul_rz(bk, d)) & 0xFFFF0000u;
#pragma unroll
            for (int c = -1; c <= 2; ++c) {
                if (c < 0 && x0 < 0x10000u) continue;
                const float x = __uint_as_float(x0 + (uint32_t)(c * 0x10000));
                // div_by_recip is the correctly rounded quotient for these d
                if (e2m1_encode1(div_by_recip(x, d, y)) != e2m1_encode1(__fmul_rn(x, yj))) ok = false;
            }
        }
        if (!ok) atomicOr(&tab.bad[j][s >> 5], 1u << (s & 31));
    }
}

// Step 3: publish ym, the first multiplier that passed.
__device__ __forceinline__ void build_qtable_m3(QTableM& tab, int tid, int nthreads) {
    for (int s = tid; s < 128; s += nthreads) {
        float ym = 0.0f;
        if (s != 0 && s < 0x7E && tab.y[s] != 0.0f) {
            for (int j = QT_NY - 1; j >= 0; --j)
                if (!((tab.bad[j][s >> 5] >> (s & 31)) & 1u)) ym = qt_multiplier(tab.y[s], j);
        }
        tab.ym[s] = ym;
    }
}

// Codes of 8 elements (4 bf16 pairs) as RN(x * y), sign included.
__device__ __forceinline__ uint32_t encode8_mul(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                                float y) {
    const uint32_t w[4] = {w0, w1, w2, w3};
    const uint64_t Y = f2pack(y, y);
    float q[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t X = f2pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
        f2unpack(mul_f32x2(X, Y), q[2 * i], q[2 * i + 1]);
    }
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return out;
}

// The divisors the multiply path rejects (and zero / saturated scales),
// kept out of line so the common path stays small.
__device__ __noinline__ uint2 quant_block16_rare(uint4 lo, uint4 hi, uint32_t sbyte, float d,
                                                 float y) {
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    uint2 r;
    if (sbyte == 0) {
        r = make_uint2(0u, 0u);
    } else if (y != 0.0f && sbyte != 0x7Eu) {
        r.x = encode8_fast(w[0], w[1], w[2], w[3], d, y);
        r.y = encode8_fast(w[4], w[5], w[6], w[7], d, y);
    } else {
        r.x = encode8(w[0], w[1], w[2], w[3], d, 0.0f, false);
        r.y = encode8(w[4], w[5], w[6], w[7], d, 0.0f, false);
    }
    return r;
}

// One 1x16 block given its max|x| bits, through QTableM.
__device__ __forceinline__ uint2 quant_block16_m(const uint32_t (&w)[8], uint32_t amax_bits,
                                                 const QTensorFast& t, const QTableM& tab,
                                                 uint32_t& sbyte) {
    sbyte = scale_byte_fast(__uint_as_float(amax_bits), t);
    const float ym = tab.ym[sbyte];
    if (ym != 0.0f) {
        uint2 r;
        r.x = encode8_mul(w[0], w[1], w[2], w[3], ym);
        r.y = encode8_mul(w[4], w[5], w[6], w[7], ym);
        return r;
    }
    return quant_block16_rare(make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]),
                              sbyte, tab.d[sbyte], tab.y[sbyte]);
}

}  // namespace ft
