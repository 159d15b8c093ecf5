// k_quant.cuh -- HBM-bound NVFP4 kernels: tensor amax, 1x16 quantization of
// activations / gradients, and the tile kernel that emits both layouts in one
// pass (16x16 weight blocks: codes packed along rows and along columns with
// one scale grid; 1x16: Q(X) and Q(X^T) sharing the tensor scale).
//
// FourTune page, section 3.2 (block-wise 16x16 weight quantization so the
// transposed weight needs no re-quantization) and section 4.3, Table 5 (1x16
// group-wise granularity).
#pragma once

#include "ft_gelu.cuh"
#include "ft_nvfp4.cuh"

namespace ft {

// ------------------------------------------------------------------ GELU
// h = GELU(y) elementwise on bf16 (ft_gelu.cuh, the table form), 8 values
// per 16-byte load; persistent CTAs, each filling its table once (its first
// loads are in flight meanwhile); n a multiple of 8, pointers 16-byte aligned.
__global__ void __launch_bounds__(1024) k_gelu_bf16(const uint16_t* __restrict__ y, uint16_t* __restrict__ h,
                                                   int64_t n) {
    __shared__ uint16_t tab[kGeluTab];
    const int64_t n8 = n / 8;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint4 v = i < n8 ? ld_nc_v4(y + 8 * i) : make_uint4(0, 0, 0, 0);
    gelu_table_build(tab, threadIdx.x, blockDim.x);
    __syncthreads();
    for (; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = i + (int64_t)gridDim.x * blockDim.x;
        const uint4 nv = j < n8 ? ld_nc_v4(y + 8 * j) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(h + 8 * i) = make_uint4(gelu_bf16x2_tab(v.x, tab), gelu_bf16x2_tab(v.y, tab),
                                                          gelu_bf16x2_tab(v.z, tab), gelu_bf16x2_tab(v.w, tab));
        v = nv;
    }
}

// ------------------------------------------------------------------ amax
// max|x| over a bf16 matrix (cols % 8 == 0, rows 16-byte aligned).  Each
// block reduces its share and folds it into the 64-bit word *out as
// (epoch << 32) | float bits with an integer atomicMax (non-negative floats
// order like their bit patterns), so the result is exact and independent of
// scheduling; the tag makes any value an earlier launch left there smaller
// than this launch's, so the word needs no clearing, and every block
// publishes, a zero block included.  The low 32 bits (the word's first four
// bytes) are then the float max|x|.  The grid is kept to a few blocks per SM
// (same-address atomics serialise in L2); each thread keeps eight 16-byte
// loads in flight.  Launched with programmatic serialization: it waits for
// the kernel before it, whose output it may read, after its own launch.
__global__ void __launch_bounds__(256) k_amax_bf16(const uint16_t* __restrict__ x, int64_t rows,
                                                   int64_t cols, int64_t ld,
                                                   unsigned long long* __restrict__ out,
                                                   unsigned long long epoch) {
    grid_dep_wait();
    constexpr int U = 8;
    const int64_t vec_per_row = cols / 8;
    const int64_t total = rows * vec_per_row;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ld == cols) {
        // software-pipelined: the next eight loads are issued before the
        // current eight are reduced, so a thread always has a batch in flight
        const uint4* xv = reinterpret_cast<const uint4*>(x);
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            v[u] = (i + u * nthr < total) ? ld_nc_v4(xv + i + u * nthr) : make_uint4(0, 0, 0, 0);
        for (; i < total; i += U * nthr) {
            const int64_t j = i + U * nthr;
            uint4 nv[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                nv[u] = (j + u * nthr < total) ? ld_nc_v4(xv + j + u * nthr) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                m = __vmaxu2(m, v[u].x & 0x7FFF7FFFu);
                m = __vmaxu2(m, v[u].y & 0x7FFF7FFFu);
                m = __vmaxu2(m, v[u].z & 0x7FFF7FFFu);
                m = __vmaxu2(m, v[u].w & 0x7FFF7FFFu);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) v[u] = nv[u];
        }
        i = total;
    }
    for (; i < total; i += nthr) {
        int64_t r = i / vec_per_row, c = i - r * vec_per_row;
        uint4 v = ld_nc_v4(x + r * ld + c * 8);
        m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    }
    m = max(m & 0xFFFFu, m >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ uint32_t red[8];
    if (lane_id() == 0) red[warp_id()] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = max(b, red[w]);
        atomicMax(out, (epoch << 32) | (unsigned long long)(b << 16));
    }
}

// ---------------------------------------------------- weight operand images
// The GEMM's image of one orientation of Q(W_res): for every 256-row tile t
// of the operand and every 256-deep stage kt of the contraction, one block
// of 288 rows of 128 bytes (36 KB): rows 0-255 hold the codes of operand
// rows 256t .. 256t + 255, contraction bytes [128 kt, 128 kt + 128); rows
// 256-287 hold the block scales of those rows for the stage in the slab
// order tensor memory wants (two 128-row halves x four 64-deep steps x 512
// bytes; byte 16l + 4i + b of a slab is the scale of half-row 32i + l, block
// b), each 16-byte chunk c of slab row p stored at chunk c ^ (p % 8) so that
// a 128-byte-swizzled copy lands it in natural order.  One copy per stage
// then brings a tile and its scales.
//   codes: the operand's codes [R, Kc/2]; grid: the 16x16 scale grid
//   [N/16, K/16]; trans = 0: operand rows are N (op_k, Kc = K), trans = 1:
//   operand rows are K (op_n, Kc = N) and the grid is read transposed.
//   rows_sc (instead of grid, for 1x16 weight groups): the operand's own
//   row-major 1x16 scales [R, Kc/16].
__global__ void __launch_bounds__(256) k_pack_wop(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ grid,
                                                  const uint8_t* __restrict__ rows_sc, int64_t N, int64_t K,
                                                  int trans, uint8_t* __restrict__ op) {
    const int64_t R = trans ? K : N, Kc = trans ? N : K;
    const int64_t KT = Kc / 256, gc = K / 16;
    const int64_t chunks = (R / 256) * KT * 288 * 8;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += nthr) {
        const int64_t blk = i / (288 * 8);
        const int rc = (int)(i - blk * 288 * 8);
        const int row = rc >> 3, c = rc & 7;
        const int64_t t = blk / KT, kt = blk - t * KT;
        uint4 v;
        if (row < 256) {
            v = *reinterpret_cast<const uint4*>(codes + (256 * t + row) * (Kc / 2) + 128 * kt + 16 * c);
        } else {
            const int pr = row - 256;
            const int nat = pr * 128 + 16 * (c ^ (pr & 7));  // natural byte offset in the scale image
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t acc = 0;
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    const int beta = nat + 4 * q + bb;
                    const int h = beta >> 11, j = (beta >> 9) & 3, e = beta & 511;
                    const int l = e >> 4, ii = (e >> 2) & 3, b = e & 3;
                    const int64_t orow = 256 * t + 128 * h + 32 * ii + l;  // operand row
                    const int64_t kb = 16 * kt + 4 * j + b;                // 16-wide contraction block
                    const uint32_t sb = rows_sc ? rows_sc[orow * (Kc / 16) + kb]
                                        : trans ? grid[kb * gc + orow / 16] : grid[(orow / 16) * gc + kb];
                    acc |= sb << (8 * bb);
                }
                w[q] = acc;
            }
            v = make_uint4(w[0], w[1], w[2], w[3]);
        }
        *reinterpret_cast<uint4*>(op + i * 16) = v;
    }
}

// ------------------------------------------------- bf16 weight images
// The 16-bit GEMMs of the precision ablation read the 4-bit weight through
// a bf16 image of one orientation: value = e2m1(code) x E4M3 block scale,
// exact in bf16 (at most 2 + 4 significant bits, exponents within range);
// the FP32 tensor scale is applied in the GEMM's epilogue, as for the 4-bit
// GEMM.  codes: [R, C/2], packed along C.  Scales: mode 0 = 16x16 grid
// [R/16, C/16]; mode 1 = 16x16 grid read transposed ([C/16, R/16], the
// codes being the grid's transposed layout); mode 2 = 1x16 row scales
// [R, C/16].  Each thread writes 8 bf16 (16 bytes) per step.
__global__ void __launch_bounds__(256) k_dequant_w(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                                   int64_t R, int64_t C, int mode, uint16_t* __restrict__ out) {
    const float e2m1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    const int64_t n8 = R * (C / 8);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / (C / 8), c = (i - r * (C / 8)) * 8;
        const uint32_t q = *reinterpret_cast<const uint32_t*>(codes + r * (C / 2) + c / 2);
        const uint32_t sb = mode == 0 ? scales[(r / 16) * (C / 16) + c / 16]
                          : mode == 1 ? scales[(c / 16) * (R / 16) + r / 16]
                                      : scales[r * (C / 16) + c / 16];
        const float sd = e4m3_decode(sb);
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t n0 = (q >> (8 * k)) & 0xFu, n1 = (q >> (8 * k + 4)) & 0xFu;
            const float v0 = __fmul_rn((n0 & 8u) ? -e2m1[n0 & 7u] : e2m1[n0 & 7u], sd);
            const float v1 = __fmul_rn((n1 & 8u) ? -e2m1[n1 & 7u] : e2m1[n1 & 7u], sd);
            const __nv_bfloat162 b = __floats2bfloat162_rn(v0, v1);
            w[k] = *reinterpret_cast<const uint32_t*>(&b);
        }
        *reinterpret_cast<uint4*>(out + r * C + c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// ------------------------------------------------------- 1x16 row-wise
// Two 16-element blocks per thread per iteration (four 16-byte loads in
// flight); stores are 8 bytes of codes and one scale byte per block;
// consecutive threads touch consecutive blocks, so accesses are coalesced.
// Many short CTAs, each with the one-step divisor table (Markstein-corrected
// quotients): measured faster here than persistent CTAs with the
// multiply-path table, whose longer build and serial loop cost more than
// the cheaper per-element encode saves.
// slab (optional, cols % 64 == 0): the scales again in the GEMM slab layout.
__global__ void __launch_bounds__(256) k_quant_1x16(const uint16_t* __restrict__ x, int64_t rows,
                                                    int64_t cols, int64_t ld,
                                                    const float* __restrict__ amax,
                                                    uint8_t* __restrict__ codes,
                                                    uint8_t* __restrict__ scales,
                                                    float* __restrict__ tscale,
                                                    uint8_t* __restrict__ slab) {
    __shared__ QTable tab;
    const QTensorFast t = make_qtensor_fast(*amax);
    build_qtable(tab, t.g, threadIdx.x, blockDim.x);
    __syncthreads();
    if (blockIdx.x == 0 && threadIdx.x == 0) *tscale = t.g;
    const int64_t nb = cols / 16;
    const int64_t total = rows * nb;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < total; b += 2 * nthr) {
        const int64_t b2 = b + nthr;
        const bool two = b2 < total;
        const int64_t r = b / nb, c = b - r * nb;
        const int64_t r2 = two ? b2 / nb : r, c2 = two ? b2 - r2 * nb : c;
        const uint16_t* p = x + r * ld + c * 16;
        const uint16_t* p2 = x + r2 * ld + c2 * 16;
        const uint4 v0 = ld_nc_v4(p), v1 = ld_nc_v4(p + 8);
        const uint4 u0 = ld_nc_v4(p2), u1 = ld_nc_v4(p2 + 8);
        uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t s;
        const uint2 q = quant_block16_fast(w, t, tab, s);
        *reinterpret_cast<uint2*>(codes + r * (cols / 2) + c * 8) = q;
        scales[r * nb + c] = (uint8_t)s;
        if (slab) slab[slab_offset(r, c, cols)] = (uint8_t)s;
        if (two) {
            uint32_t w2[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            const uint2 q2 = quant_block16_fast(w2, t, tab, s);
            *reinterpret_cast<uint2*>(codes + r2 * (cols / 2) + c2 * 8) = q2;
            scales[r2 * nb + c2] = (uint8_t)s;
            if (slab) slab[slab_offset(r2, c2, cols)] = (uint8_t)s;
        }
    }
}

// ---------------------------------------------------- tile kernel (both layouts)
// Persistent CTAs over 64 x 128 tiles of x (a 16-wide block never straddles
// a tile edge: rows and cols are multiples of 16).  A tile is read once with
// coalesced 16-byte loads into shared memory (rows padded to 272 bytes, so
// the column pass reads conflict-free), then:
//   row pass    thread t takes blocks (row, b) = (j / 8, j % 8) for j = t and
//               t + 256: a warp covers 4 rows x 8 blocks, so its 8-byte code
//               stores fill whole 64-byte row pieces;
//   column pass thread t takes columns 2 (t % 64) and 2 (t % 64) + 1, rows
//               16 (t / 64) .. + 15; column codes and scales are staged in
//               shared memory and leave as 32-byte column pieces (16-byte
//               stores) and 4-byte scale words.
// kMode16x16 = true : one scale per 16x16 tile (weights).  Writes codes
//   packed along rows (codes_row, [rows, cols/2]) and, if codes_col !=
//   nullptr, the same codes packed along columns ([cols, rows/2]) -- the
//   nibbles transposed through shared memory, no second encode; scale grid
//   [rows/16, cols/16].
// kMode16x16 = false: 1x16 blocks (activations).  Row blocks -> codes_row /
//   scales_row ([rows, cols/16]); column blocks (16 consecutive rows of one
//   column) -> codes_col / scales_col ([cols, rows/16]); both share g.
constexpr int QTT_R = 64, QTT_C = 128;
constexpr int QTT_LDW = QTT_C / 2 + 4;  // shared row stride in words (272 bytes)

struct QTileSmem {
    uint32_t x[QTT_R * QTT_LDW];  // the tile, bf16 pairs
    uint8_t crow[QTT_R * 64];     // 16x16 mode: the row codes, for the transpose
    uint8_t ccol[QTT_C * 32];     // column codes, 32 bytes (64 rows) per column
    uint8_t cscale[QTT_C * 4];    // 1x16 mode: column scales, 4 per column
    uint32_t rbmax[QTT_R * 8];    // 16x16 mode: max bits of each row block
    uint32_t tmax[4 * 8];         // 16x16 mode: max bits of each 16x16 tile
    QTableM tab;
};

template <bool kMode16x16>
__global__ void __launch_bounds__(256) k_quant_tile16(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    const float* __restrict__ amax, uint8_t* __restrict__ codes_row,
    uint8_t* __restrict__ scales_row, uint8_t* __restrict__ codes_col,
    uint8_t* __restrict__ scales_col, float* __restrict__ tscale, float* __restrict__ tscale2) {
    __shared__ __align__(16) QTileSmem sm;
    const QTensorFast qt = make_qtensor_fast(*amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *tscale = qt.g;
        if (tscale2) *tscale2 = qt.g;
    }
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t ntc = (cols + QTT_C - 1) / QTT_C;
    const int64_t ntiles = ((rows + QTT_R - 1) / QTT_R) * ntc;
    const uint32_t xs = smem_u32(sm.x);
    // whole-word stores are aligned only for these shapes; else byte stores
    const bool rs8 = (cols % QTT_C) == 0;   // 8 row scales of a tile row: one 8-byte store
    const bool cc16 = (rows % 32) == 0;     // column codes: 16-byte pieces
    const bool cs4 = (rows % QTT_R) == 0;   // column scales: 4-byte words

    for (int64_t ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
        const int64_t r0 = (ti / ntc) * QTT_R, c0 = (ti % ntc) * QTT_C;
        const int vr = (int)min((int64_t)QTT_R, rows - r0);  // multiples of 16
        const int vc = (int)min((int64_t)QTT_C, cols - c0);
        __syncthreads();  // the previous tile's shared reads are done
        {
            uint4 v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = tid + 256 * k, r = i >> 4, ch = i & 15;
                v[k] = (r < vr && 8 * ch < vc) ? ld_nc_v4(x + (r0 + r) * ld + c0 + 8 * ch) : make_uint4(0, 0, 0, 0);
            }
            if (ti == blockIdx.x) {
                // the encode table, built while the first tile's loads are in flight
                build_qtable_m1(sm.tab, qt.g, tid, blockDim.x);
                __syncthreads();
                build_qtable_m2(sm.tab, tid, blockDim.x);
                __syncthreads();
                build_qtable_m3(sm.tab, tid, blockDim.x);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = tid + 256 * k, r = i >> 4, ch = i & 15;
                st_shared_v4(xs + (uint32_t)(r * QTT_LDW + 4 * ch) * 4u, v[k]);
            }
        }
        __syncthreads();

        // ---------------- row pass
        uint32_t w[2][8];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int j = tid + 256 * k, row = j >> 3, b = j & 7;
            const uint32_t a = xs + (uint32_t)(row * QTT_LDW + 8 * b) * 4u;
            const uint4 lo = ld_shared_v4(a), hi = ld_shared_v4(a + 16);
            w[k][0] = lo.x; w[k][1] = lo.y; w[k][2] = lo.z; w[k][3] = lo.w;
            w[k][4] = hi.x; w[k][5] = hi.y; w[k][6] = hi.z; w[k][7] = hi.w;
        }
        if (kMode16x16) {
#pragma unroll
            for (int k = 0; k < 2; ++k) sm.rbmax[tid + 256 * k] = amax_bits_16(w[k]);
            __syncthreads();
            if (tid < 32) {
                const int tr = tid >> 3, tc = tid & 7;
                uint32_t m = 0;
#pragma unroll
                for (int i = 0; i < 16; ++i) m = max(m, sm.rbmax[(16 * tr + i) * 8 + tc]);
                sm.tmax[tid] = m;
            }
            __syncthreads();
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int j = tid + 256 * k, row = j >> 3, b = j & 7;
            const bool valid = row < vr && 16 * b < vc;
            uint32_t sbyte;
            const uint32_t mbits = kMode16x16 ? sm.tmax[(row >> 4) * 8 + b] : amax_bits_16(w[k]);
            const uint2 q = quant_block16_m(w[k], mbits, qt, sm.tab, sbyte);
            if (valid) *reinterpret_cast<uint2*>(codes_row + (r0 + row) * (cols / 2) + c0 / 2 + 8 * b) = q;
            if (kMode16x16) {
                *reinterpret_cast<uint2*>(sm.crow + row * 64 + 8 * b) = q;
                if (valid && (row & 15) == 0) scales_row[((r0 + row) >> 4) * (cols / 16) + c0 / 16 + b] = (uint8_t)sbyte;
            } else {
                // the 8 scale bytes of a row are lanes 8 (row % 4) .. + 7
                uint32_t sv = sbyte << (8 * (b & 3));
                sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 1);
                sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 2);
                const uint32_t hi = __shfl_down_sync(0xFFFFFFFFu, sv, 4);
                uint8_t* srow = scales_row + (r0 + row) * (cols / 16) + c0 / 16;
                if (rs8 && vc == QTT_C) {
                    if (b == 0 && row < vr) *reinterpret_cast<uint2*>(srow) = make_uint2(sv, hi);
                } else if (valid) {
                    srow[b] = (uint8_t)sbyte;
                }
            }
        }
        (void)lane;
        if (kMode16x16 && !codes_col) continue;
        if (kMode16x16) __syncthreads();  // the row codes are staged

        // ---------------- column pass: columns 2 cp, 2 cp + 1, rows 16 rb ..
        {
            const int cp = tid & 63, rb = tid >> 6;
            uint2 q0 = make_uint2(0u, 0u), q1 = make_uint2(0u, 0u);
            uint32_t s0 = 0, s1 = 0;
            if (kMode16x16) {
                // transpose the nibbles: byte cp of a row holds columns 2 cp
                // (low nibble) and 2 cp + 1 (high nibble)
                uint32_t e[4] = {0, 0, 0, 0}, o[4] = {0, 0, 0, 0};
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t byte = sm.crow[(16 * rb + i) * 64 + cp];
                    e[i >> 2] |= (byte & 0xFu) << (4 * (i & 7));
                    o[i >> 2] |= (byte >> 4) << (4 * (i & 7));
                }
                q0 = make_uint2(e[0] | e[1], e[2] | e[3]);
                q1 = make_uint2(o[0] | o[1], o[2] | o[3]);
            } else {
                uint32_t wc[2][8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t a = sm.x[(16 * rb + 2 * i) * QTT_LDW + cp];
                    const uint32_t b = sm.x[(16 * rb + 2 * i + 1) * QTT_LDW + cp];
                    wc[0][i] = __byte_perm(a, b, 0x5410);  // column 2 cp, rows 2i, 2i + 1
                    wc[1][i] = __byte_perm(a, b, 0x7632);  // column 2 cp + 1
                }
                q0 = quant_block16_m(wc[0], amax_bits_16(wc[0]), qt, sm.tab, s0);
                q1 = quant_block16_m(wc[1], amax_bits_16(wc[1]), qt, sm.tab, s1);
                sm.cscale[(2 * cp) * 4 + rb] = (uint8_t)s0;
                sm.cscale[(2 * cp + 1) * 4 + rb] = (uint8_t)s1;
            }
            *reinterpret_cast<uint2*>(sm.ccol + (2 * cp) * 32 + 8 * rb) = q0;
            *reinterpret_cast<uint2*>(sm.ccol + (2 * cp + 1) * 32 + 8 * rb) = q1;
        }
        __syncthreads();
        {
            // column c's 32 code bytes (64 rows): two 16-byte pieces
            const int c = tid >> 1, h = tid & 1;
            if (c < vc) {
                uint8_t* dst = codes_col + (c0 + c) * (rows / 2) + r0 / 2 + 16 * h;
                const uint8_t* src = sm.ccol + c * 32 + 16 * h;
                if (cc16 && 32 * h + 32 <= vr) {
                    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
                } else {
#pragma unroll
                    for (int k = 0; k < 2; ++k)
                        if (32 * h + 16 * k < vr)
                            *reinterpret_cast<uint2*>(dst + 8 * k) = *reinterpret_cast<const uint2*>(src + 8 * k);
                }
            }
            if (!kMode16x16 && tid < QTT_C && tid < vc) {
                uint8_t* dst = scales_col + (c0 + tid) * (rows / 16) + r0 / 16;
                if (cs4 && vr == QTT_R) {
                    *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(sm.cscale + tid * 4);
                } else {
                    for (int k = 0; 16 * k < vr; ++k) dst[k] = sm.cscale[tid * 4 + k];
                }
            }
        }
    }
}

}  // namespace ft
