/*
 * ft_oracle.c -- plain, slow, obviously-correct CPU oracle for the W4A4G4
 * triple-branch linear layer of "FourTune: Towards Fully 4-Bit Efficient
 * Post-Training for Diffusion Models".
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline leg use it.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * What it implements (bit level, from the format definitions):
 *   - E2M1 (4-bit float: 1 sign, 2 exponent, 1 mantissa bit) encode/decode.
 *   - E4M3 (8-bit float, finite-only "fn" variant, max 448) encode/decode.
 *   - NVFP4 block quantization with a FP32 tensor scale: 1x16 blocks along the
 *     contiguous axis (activations, gradients) and 16x16 blocks (weights).
 *     FourTune page, section 3.2 "4-Bit Backward Pass via Block-Quantization"
 *     (16x16 weight blocks so the transposed weight needs no re-quantization)
 *     and section 4.3 / Table 5 (1x16 "group-wise" granularity).
 *     The generic quantizer W~ = Round(W / s) is the one of section 2.3.
 *
 * The encode step follows these readings (the page only says "NVFP4"):
 *   g   = amax_tensor / 2688           (FP32 decode scale; g = 1 if amax = 0)
 *   sf  = amax_block / (6 * g)         (FP32: product rounded, then quotient)
 *   s   = E4M3_RNE_satfinite(sf)       (stored byte; sd = its value)
 *   q   = x / (sd * g)                 (FP32: product rounded, then quotient)
 *   c   = E2M1_RNE_satfinite(q)        (sign kept; sd == 0 gives code 0)
 *   deq = e2m1(c) * sd * g             (exact in FP64)
 * Two codes per byte, lower-index element in the low nibble.
 *
 * Arithmetic is IEEE single precision with round-to-nearest-even; the build
 * uses -ffp-contract=off and no fast-math, so no FMA contraction and
 * denormals are kept.
 *
 * Encoders pick the nearest representable value by plain comparison against
 * the table of all representable magnitudes; equidistant candidates resolve
 * to the even code (the one whose lowest mantissa bit is 0).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

/* ---------------------------------------------------------------- formats */

/* E2M1 magnitudes, code 0..7: exponent bias 1, one mantissa bit.
 * e=0: subnormal 0, 0.5; e=1: 1, 1.5; e=2: 2, 3; e=3: 4, 6. */
static const double kE2M1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double fto_e2m1_value(uint8_t code) {
    double m = kE2M1Mag[code & 7u];
    return (code & 8u) ? -m : m;
}

/* Nearest E2M1 magnitude, ties to the even code; anything above 6 saturates
 * to 6 (the nearest grid point of a value beyond the top is the top). */
uint8_t fto_e2m1_encode(float q) {
    uint8_t sign = signbit(q) ? 8u : 0u;
    double a = fabs((double)q);
    if (a >= 6.0) return (uint8_t)(sign | 7u); /* saturation, infinity included */
    int best = 0;
    double best_d = a; /* distance to magnitude 0 */
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - kE2M1Mag[c]);
        if (d < best_d || (d == best_d && (c % 2) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | (uint8_t)best);
}

/* E4M3 (fn) value of a byte: 1 sign, 4 exponent bits (bias 7), 3 mantissa.
 * Exponent field 0 is subnormal (m * 2^-9).  0x7F / 0xFF are NaN. */
double fto_e4m3_value(uint8_t byte) {
    int s = (byte >> 7) & 1;
    int e = (byte >> 3) & 0xF;
    int m = byte & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* E4M3 round-to-nearest-even with saturation to +-448 (satfinite).
 * The non-negative finite codes 0x00..0x7E are monotone in value, so the
 * nearest code is found among the two table entries that bracket |v|. */
uint8_t fto_e4m3_encode(float v) {
    uint8_t sign = signbit(v) ? 0x80u : 0u;
    double a = fabs((double)v);
    if (isnan(v)) return (uint8_t)(sign | 0x7Fu);
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);
    /* largest code lo with value(lo) <= a */
    int lo = 0;
    for (int c = 0; c <= 0x7E; ++c)
        if (fto_e4m3_value((uint8_t)c) <= a) lo = c;
    int hi = lo + 1; /* value(hi) > a, hi <= 0x7E because a < 448 */
    double dlo = a - fto_e4m3_value((uint8_t)lo);
    double dhi = fto_e4m3_value((uint8_t)hi) - a;
    int pick;
    if (dlo < dhi) pick = lo;
    else if (dhi < dlo) pick = hi;
    else pick = (lo % 2 == 0) ? lo : hi;
    return (uint8_t)(sign | (uint8_t)pick);
}

/* bf16 bit pattern -> float (exact widening). */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ----------------------------------------------------------- tensor scale */

/* max |x| over a rows x cols bf16 matrix with leading dimension ld. */
float fto_amax_bf16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld) {
    float m = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(bf16_to_f32(x[r * ld + c]));
            if (a > m) m = a;
        }
    return m;
}

/* Decode tensor scale g = amax / (6 * 448), 1 for an all-zero tensor. */
float fto_tensor_scale(float amax) {
    if (amax == 0.0f) return 1.0f;
    volatile float denom = 2688.0f;
    return amax / denom;
}

/* One block: given its amax and the tensor scale, the E4M3 scale byte. */
static uint8_t block_scale_byte(float amax_b, float g) {
    volatile float six_g = 6.0f * g;  /* rounded product */
    volatile float sf = amax_b / six_g;
    return fto_e4m3_encode(sf);
}

/* One element: code given the scale byte value sd and tensor scale g. */
static uint8_t element_code(float x, float sd, float g) {
    if (sd == 0.0f) return 0u;
    volatile float d = sd * g;  /* rounded product */
    volatile float q = x / d;   /* rounded quotient */
    return fto_e2m1_encode(q);
}

static void put_nibble(uint8_t* row, int64_t idx, uint8_t code) {
    uint8_t* b = &row[idx / 2];
    if ((idx & 1) == 0)
        *b = (uint8_t)((*b & 0xF0u) | (code & 0xFu));
    else
        *b = (uint8_t)((*b & 0x0Fu) | (uint8_t)((code & 0xFu) << 4));
}

static uint8_t get_nibble(const uint8_t* row, int64_t idx) {
    uint8_t b = row[idx / 2];
    return (idx & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0xFu);
}

/* ------------------------------------------------------ 1x16 quantization */

/* Quantize a rows x cols bf16 matrix in 1x16 blocks along the row.
 * amax: the tensor amax to use (pass a negative value to compute it).
 * codes: rows x cols/2 bytes (row-major); scales: rows x cols/16 bytes.
 * Returns the tensor scale g through *g_out.  cols must be a multiple of 16. */
void fto_quantize_1x16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                       float amax, uint8_t* codes, uint8_t* scales, float* g_out) {
    if (amax < 0.0f) amax = fto_amax_bf16(x, rows, cols, ld);
    float g = fto_tensor_scale(amax);
    *g_out = g;
    int64_t nb = cols / 16;
    for (int64_t r = 0; r < rows; ++r) {
        uint8_t* crow = codes + r * (cols / 2);
        for (int64_t b = 0; b < nb; ++b) {
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(bf16_to_f32(x[r * ld + b * 16 + i]));
                if (a > amax_b) amax_b = a;
            }
            uint8_t s = block_scale_byte(amax_b, g);
            scales[r * nb + b] = s;
            float sd = (float)fto_e4m3_value(s);
            for (int i = 0; i < 16; ++i) {
                float xv = bf16_to_f32(x[r * ld + b * 16 + i]);
                put_nibble(crow, b * 16 + i, element_code(xv, sd, g));
            }
        }
    }
}

/* ---------------------------------------------------- 16x16 quantization */

/* Quantize a rows x cols bf16 matrix in 16x16 blocks.
 * codes_row: rows x cols/2 (codes packed along a row);
 * codes_col: cols x rows/2 (the same codes, transposed: packed along a column),
 *            may be NULL;
 * scales: (rows/16) x (cols/16) grid, one byte per 16x16 block. */
void fto_quantize_16x16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                        float amax, uint8_t* codes_row, uint8_t* codes_col,
                        uint8_t* scales, float* g_out) {
    if (amax < 0.0f) amax = fto_amax_bf16(x, rows, cols, ld);
    float g = fto_tensor_scale(amax);
    *g_out = g;
    int64_t br = rows / 16, bc = cols / 16;
    for (int64_t i = 0; i < br; ++i)
        for (int64_t j = 0; j < bc; ++j) {
            float amax_b = 0.0f;
            for (int u = 0; u < 16; ++u)
                for (int v = 0; v < 16; ++v) {
                    float a = fabsf(bf16_to_f32(x[(i * 16 + u) * ld + j * 16 + v]));
                    if (a > amax_b) amax_b = a;
                }
            uint8_t s = block_scale_byte(amax_b, g);
            scales[i * bc + j] = s;
            float sd = (float)fto_e4m3_value(s);
            for (int u = 0; u < 16; ++u)
                for (int v = 0; v < 16; ++v) {
                    int64_t r = i * 16 + u, c = j * 16 + v;
                    uint8_t code = element_code(bf16_to_f32(x[r * ld + c]), sd, g);
                    put_nibble(codes_row + r * (cols / 2), c, code);
                    if (codes_col) put_nibble(codes_col + c * (rows / 2), r, code);
                }
        }
}

/* ------------------------------------------------------------ dequantize */

/* 1x16: out[r*cols + c] = e2m1(code) * sd(scale of block c/16) * g. */
void fto_dequant_1x16(const uint8_t* codes, const uint8_t* scales, float g,
                      int64_t rows, int64_t cols, double* out) {
    int64_t nb = cols / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            double sd = fto_e4m3_value(scales[r * nb + c / 16]);
            out[r * cols + c] =
                fto_e2m1_value(get_nibble(codes + r * (cols / 2), c)) * sd * (double)g;
        }
}

/* 16x16 (row layout): scale of element (r, c) is grid[r/16][c/16]. */
void fto_dequant_16x16(const uint8_t* codes_row, const uint8_t* scales, float g,
                       int64_t rows, int64_t cols, double* out) {
    int64_t bc = cols / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            double sd = fto_e4m3_value(scales[(r / 16) * bc + c / 16]);
            out[r * cols + c] =
                fto_e2m1_value(get_nibble(codes_row + r * (cols / 2), c)) * sd * (double)g;
        }
}

/* Plain FP64 product C[i,j] = sum_k A[i,k] * B[j,k] (both row-major, K
 * contiguous), for the rows listed in row_idx (n_rows of them).  Used to pin
 * the library matmul the Python side uses, on small cases. */
void fto_gemm_nt_f64(const double* A, const double* B, int64_t K, int64_t N,
                     const int64_t* row_idx, int64_t n_rows, double* C) {
    for (int64_t t = 0; t < n_rows; ++t) {
        const double* a = A + row_idx[t] * K;
        for (int64_t j = 0; j < N; ++j) {
            const double* b = B + j * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += a[k] * b[k];
            C[t * N + j] = acc;
        }
    }
}
