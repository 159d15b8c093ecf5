// k_qdown.cuh -- LoRA fusion, down side (FourTune page, section 3.3: all
// three branches share the input, so quantization and the down-projections
// run as one kernel that reads the input once).
//
// For an input T [M, C] (X in the forward, dY in the backward) one pass
// emits
//   Q(T)  : 1x16 NVFP4 codes [M, C/2] and scales [M, C/16]
//   part  : FP32 partial sums of T @ [L1 | L2] over this CTA's C-range,
//           [splits, M, r]; k_lowrank_finalize adds the splits in a fixed
//           order and rounds  P = [bf16(T L1) | bf16(s T L2)].
// The down-projection runs on tcgen05 (kind::f16, bf16 in, f32 in TMEM) with
// the roles swapped so the rank is the MMA's M:  D[j, m] = sum_c Lt[j, c]
// T[m, c], where Lt = [L1 | L2]^T zero-padded to 128 rows (k_pack_lt).
//
// CTA = 128 rows of T x one C-range; warps: 0 TMA producer, 1 UMMA issuer,
// 2-5 quantizers (thread t owns row t of each 128 x 64 stage, read from the
// same swizzled shared-memory tile the MMA consumes) and epilogue.
#pragma once

#include <cuda.h>

#include "ft_nvfp4.cuh"

namespace ft {
namespace qdown {

constexpr int BM = 128;
constexpr int BKC = 64;  // columns of T per stage (128 bytes of bf16)
constexpr int STAGES = 4;
constexpr int NUM_THREADS = 192;
constexpr int TILE_BYTES = BM * BKC * 2;  // 16 KiB
constexpr uint32_t TMEM_COLS = 128;

struct Params {
    CUtensorMap mapT;   // bf16 [M, C], box {64, 128}, 128 B swizzle
    CUtensorMap mapLt;  // bf16 [128, C], box {64, 128}, 128 B swizzle
    const float* amax;
    float* tscale;
    uint8_t* codes;
    uint8_t* scales;
    float* part;
    int M, C, r, cchunk;
    int do_mma;
};

constexpr uint32_t SMEM_BYTES = STAGES * 2 * TILE_BYTES + 256 + 1024;

__global__ void __launch_bounds__(NUM_THREADS, 1) k_qdown(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const uint32_t off_x = 0, off_l = STAGES * TILE_BYTES, off_bar = 2 * STAGES * TILE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + off_bar);
    uint64_t* empty = full + STAGES;
    uint64_t* accfull = empty + STAGES;
    uint64_t* drain = accfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();
    const int m0 = blockIdx.x * BM;
    const int split = blockIdx.y;
    const int c0 = split * p.cchunk;
    const int cn = min(p.cchunk, p.C - c0);
    const int nst = cn / BKC;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 4 + (p.do_mma ? 1 : 0));
        }
        mbar_init(accfull, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1 && p.do_mma) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = p.do_mma ? *tmem_slot : 0u;

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t bytes = TILE_BYTES * (p.do_mma ? 2u : 1u);
            int st = 0;
            for (; st < nst; ++st) {
                const int s = st % STAGES;
                const uint32_t ph = (st / STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, ERR_WAIT_EMPTY, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(smem + off_x + s * TILE_BYTES, &p.mapT, &full[s], c0 + st * BKC, m0);
                if (p.do_mma)
                    tma_load_2d(smem + off_l + s * TILE_BYTES, &p.mapLt, &full[s], c0 + st * BKC, 0);
            }
            if (st < nst) {
                for (int d = 0; d < STAGES && d < st; ++d) {
                    int j = st - 1 - d;
                    volatile int no_abort = 0;
                    mbar_wait(&full[j % STAGES], (j / STAGES) & 1, ERR_WAIT_DRAIN, &no_abort);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && p.do_mma) {
            const uint32_t idesc = idesc_bf16(128, BM, 0, 0);
            bool ok = true;
            for (int st = 0; st < nst; ++st) {
                const int s = st % STAGES;
                const uint32_t ph = (st / STAGES) & 1;
                if (!mbar_wait(&full[s], ph, ERR_WAIT_FULL, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a = base + off_l + s * TILE_BYTES;
                const uint32_t b = base + off_x + s * TILE_BYTES;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_bf16(tmem, desc_kmajor_sw128(a + 32 * j), desc_kmajor_sw128(b + 32 * j), idesc,
                              (st | j) != 0);
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(accfull);
            tc_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, ERR_WAIT_DRAIN, &no_abort);
        }
        __syncwarp();
    } else {
        // quantizers: thread t owns row t of the tile
        const int t = threadIdx.x - 64;
        const int row = m0 + t;
        const QTensor qt = make_qtensor(*p.amax);
        if (blockIdx.x == 0 && blockIdx.y == 0 && t == 0) *p.tscale = qt.g;
        bool ok = true;
        const uint32_t sw = (uint32_t)(t & 7);
        for (int st = 0; st < nst; ++st) {
            const int s = st % STAGES;
            const uint32_t ph = (st / STAGES) & 1;
            if (!mbar_wait(&full[s], ph, ERR_WAIT_FULL, abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t rowaddr = base + off_x + s * TILE_BYTES + t * 128;
            uint32_t codes_out[8];
            uint32_t sc = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                uint4 v0 = ld_shared_v4(rowaddr + (((2 * b) ^ sw) << 4));
                uint4 v1 = ld_shared_v4(rowaddr + (((2 * b + 1) ^ sw) << 4));
                uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                uint32_t sbyte;
                uint2 q = quant_block16(w, qt, sbyte);
                codes_out[2 * b] = q.x;
                codes_out[2 * b + 1] = q.y;
                sc |= sbyte << (8 * b);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (row < p.M) {
                const int col = c0 + st * BKC;
                uint4* cdst = reinterpret_cast<uint4*>(p.codes + (int64_t)row * (p.C / 2) + col / 2);
                cdst[0] = make_uint4(codes_out[0], codes_out[1], codes_out[2], codes_out[3]);
                cdst[1] = make_uint4(codes_out[4], codes_out[5], codes_out[6], codes_out[7]);
                *reinterpret_cast<uint32_t*>(p.scales + (int64_t)row * (p.C / 16) + col / 16) = sc;
            }
        }
        if (p.do_mma && ok) {
            // epilogue: TMEM lane = rank index j, column = tile row
            if (mbar_wait(accfull, 0, ERR_WAIT_ACC_FULL, abort_flag)) {
                tc_fence_after();
                const int sp = warp & 3;
                const int j = 32 * sp + lane;
                const uint32_t lane_addr = (uint32_t)(32 * sp) << 16;
#pragma unroll 1
                for (int c = 0; c < BM / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + lane_addr + 32 * c, v);
                    tmem_ld_wait();
                    if (j < p.r) {
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const int m = m0 + 32 * c + k;
                            if (m < p.M)
                                p.part[((int64_t)split * p.M + m) * p.r + j] = __uint_as_float(v[k]);
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && p.do_mma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace qdown

// Lt[j, c] = L1[c, j] (j < r1), L2[c, j - r1] (j < r1 + r2), 0 (j < 128):
// the transposed, zero-padded low-rank factor the down-projection MMA reads.
__global__ void __launch_bounds__(256) k_pack_lt(const uint16_t* __restrict__ L1, int r1,
                                                 const uint16_t* __restrict__ L2, int r2, int C,
                                                 uint16_t* __restrict__ Lt) {
    const int64_t total = (int64_t)128 * C;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int j = (int)(i / C);
        const int c = (int)(i - (int64_t)j * C);
        uint16_t v = 0;
        if (j < r1)
            v = L1[(int64_t)c * r1 + j];
        else if (j < r1 + r2)
            v = L2[(int64_t)c * r2 + (j - r1)];
        Lt[i] = v;
    }
}

// P[m, j] = bf16( sum_split part[split, m, j] * (j < r1 ? 1 : s) ), splits
// added in increasing order.
__global__ void __launch_bounds__(256) k_lowrank_finalize(const float* __restrict__ part, int splits,
                                                          int M, int r, int r1, float s,
                                                          __nv_bfloat16* __restrict__ P) {
    const int64_t total = (int64_t)M * r;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.0f;
        for (int k = 0; k < splits; ++k) acc = __fadd_rn(acc, part[(int64_t)k * total + i]);
        const int j = (int)(i % r);
        if (j >= r1) acc = __fmul_rn(acc, s);
        P[i] = __float2bfloat16_rn(acc);
    }
}

}  // namespace ft
