// k_quant.cuh -- HBM-bound NVFP4 kernels: tensor amax, 1x16 quantization of
// activations / gradients, and the tile kernel that emits both layouts in one
// pass (16x16 weight blocks: codes packed along rows and along columns with
// one scale grid; 1x16: Q(X) and Q(X^T) sharing the tensor scale).
//
// FourTune page, section 3.2 (block-wise 16x16 weight quantization so the
// transposed weight needs no re-quantization) and section 4.3, Table 5 (1x16
// group-wise granularity).
#pragma once

#include "ft_nvfp4.cuh"

namespace ft {

// ------------------------------------------------------------------ amax
// max|x| over a bf16 matrix (cols % 8 == 0, rows 16-byte aligned).  Each
// block reduces its share and folds it into *out with an integer atomicMax on
// the float bits (non-negative floats order like their bit patterns), so the
// result is exact and independent of scheduling.  *out must be 0 on entry.
// The grid is kept to a few blocks per SM (same-address atomics serialise in
// L2); each thread keeps eight independent 16-byte loads in flight.
__global__ void __launch_bounds__(256) k_amax_bf16(const uint16_t* __restrict__ x, int64_t rows,
                                                   int64_t cols, int64_t ld,
                                                   unsigned int* __restrict__ out) {
    constexpr int U = 8;
    const int64_t vec_per_row = cols / 8;
    const int64_t total = rows * vec_per_row;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (ld == cols) {
        const uint4* xv = reinterpret_cast<const uint4*>(x);
        for (; i < total; i += U * nthr) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                v[u] = (i + u * nthr < total) ? ld_nc_v4(xv + i + u * nthr) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                m = __vmaxu2(m, v[u].x & 0x7FFF7FFFu);
                m = __vmaxu2(m, v[u].y & 0x7FFF7FFFu);
                m = __vmaxu2(m, v[u].z & 0x7FFF7FFFu);
                m = __vmaxu2(m, v[u].w & 0x7FFF7FFFu);
            }
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
        if (b) atomicMax(out, b << 16);
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

// ------------------------------------------------------- 1x16 row-wise
// Two 16-element blocks per thread per iteration (four 16-byte loads in
// flight); stores are 8 bytes of codes and one scale byte per block;
// consecutive threads touch consecutive blocks, so accesses are coalesced.
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

// ---------------------------------------------------- 16x16 tile kernel
// One warp per 16x16 tile.  Lane l holds row (l & 15), columns 8*(l >> 4)
// .. +7 of the tile (one 16-byte load).
//
// kMode16x16 = true : one scale per tile (weights).  Writes codes packed
//   along rows (codes_row, [rows, cols/2]) and, if codes_col != nullptr,
//   the same codes packed along columns ([cols, rows/2]); scale grid
//   [rows/16, cols/16].
// kMode16x16 = false: 1x16 blocks (activations).  Row blocks -> codes_row /
//   scales_row ([rows, cols/16]); column blocks (16 consecutive rows of one
//   column) -> codes_col / scales_col ([cols, rows/16]); both share g.
template <bool kMode16x16>
__global__ void __launch_bounds__(256) k_quant_tile16(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    const float* __restrict__ amax, uint8_t* __restrict__ codes_row,
    uint8_t* __restrict__ scales_row, uint8_t* __restrict__ codes_col,
    uint8_t* __restrict__ scales_col, float* __restrict__ tscale, float* __restrict__ tscale2) {
    __shared__ uint32_t tile[8][16][9];  // per warp: 16 rows x 8 bf16 pairs (+1 pad)
    const QTensor t = make_qtensor(*amax);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        *tscale = t.g;
        if (tscale2) *tscale2 = t.g;
    }
    const int w = warp_id(), l = lane_id();
    const int64_t tiles_c = cols / 16;
    const int64_t tr = blockIdx.y;                            // tile row
    const int64_t tc = (int64_t)blockIdx.x * 8 + w;           // tile column
    if (tc >= tiles_c) return;
    const int r = l & 15, h = l >> 4;
    const int64_t row = tr * 16 + r;
    const int64_t col = tc * 16 + h * 8;
    uint4 v = ld_nc_v4(x + row * ld + col);
    uint32_t mine[4] = {v.x, v.y, v.z, v.w};

    if (kMode16x16) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) m = __vmaxu2(m, mine[i] & 0x7FFF7FFFu);
        m = max(m & 0xFFFFu, m >> 16);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        float amax_b = __uint_as_float(m << 16);
        uint32_t s;
        BlockDiv bd;
        uint32_t code8 = 0;
        if (block_divisor(amax_b, t, s, bd))
            code8 = encode8(mine[0], mine[1], mine[2], mine[3], bd.d, bd.y, bd.fast);
        *reinterpret_cast<uint32_t*>(codes_row + row * (cols / 2) + col / 2) = code8;
        if (l == 0) scales_row[tr * tiles_c + tc] = (uint8_t)s;
        if (codes_col) {
            // transpose the 16x16 nibble tile through shared memory
            uint32_t* tw = &tile[w][0][0];
            tw[r * 9 + h] = code8;  // row r, columns 8h..8h+7 (nibbles)
            __syncwarp();
            // lane l: column c = l & 15, rows 8*(l>>4) .. +7
            const int c = l & 15, rh = l >> 4;
            uint32_t out = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int rr = rh * 8 + i;
                uint32_t word = tw[rr * 9 + (c >> 3)];
                uint32_t nib = (word >> (4 * (c & 7))) & 0xFu;
                out |= nib << (4 * i);
            }
            *reinterpret_cast<uint32_t*>(codes_col + (tc * 16 + c) * (rows / 2) + tr * 8 + rh * 4) =
                out;
        }
    } else {
        // row blocks: lanes r and r+16 hold the two halves of row r
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) m = __vmaxu2(m, mine[i] & 0x7FFF7FFFu);
        m = max(m & 0xFFFFu, m >> 16);
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
        {
            float amax_b = __uint_as_float(m << 16);
            uint32_t s;
            BlockDiv bd;
            uint32_t code8 = 0;
            if (block_divisor(amax_b, t, s, bd))
                code8 = encode8(mine[0], mine[1], mine[2], mine[3], bd.d, bd.y, bd.fast);
            *reinterpret_cast<uint32_t*>(codes_row + row * (cols / 2) + col / 2) = code8;
            if (h == 0) scales_row[row * tiles_c + tc] = (uint8_t)s;
        }
        // column blocks: gather column c (rows 8h'..8h'+7) through shared memory
        uint32_t* tw = &tile[w][0][0];
#pragma unroll
        for (int i = 0; i < 4; ++i) tw[r * 9 + h * 4 + i] = mine[i];
        __syncwarp();
        const int c = l & 15, rh = l >> 4;
        uint32_t cw[4];  // 8 bf16 of column c, rows rh*8 .. +7, packed in pairs
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int r0 = rh * 8 + 2 * i;
            uint32_t a = tw[r0 * 9 + (c >> 1)];
            uint32_t b = tw[(r0 + 1) * 9 + (c >> 1)];
            uint32_t ea = (c & 1) ? (a >> 16) : (a & 0xFFFFu);
            uint32_t eb = (c & 1) ? (b >> 16) : (b & 0xFFFFu);
            cw[i] = ea | (eb << 16);
        }
        uint32_t mc = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) mc = __vmaxu2(mc, cw[i] & 0x7FFF7FFFu);
        mc = max(mc & 0xFFFFu, mc >> 16);
        mc = max(mc, __shfl_xor_sync(0xFFFFFFFFu, mc, 16));
        float amax_c = __uint_as_float(mc << 16);
        uint32_t s;
        BlockDiv bd;
        uint32_t code8 = 0;
        if (block_divisor(amax_c, t, s, bd)) code8 = encode8(cw[0], cw[1], cw[2], cw[3], bd.d, bd.y, bd.fast);
        const int64_t ccol = tc * 16 + c;
        *reinterpret_cast<uint32_t*>(codes_col + ccol * (rows / 2) + tr * 8 + rh * 4) = code8;
        if (rh == 0) scales_col[ccol * (rows / 16) + tr] = (uint8_t)s;
    }
}

}  // namespace ft
