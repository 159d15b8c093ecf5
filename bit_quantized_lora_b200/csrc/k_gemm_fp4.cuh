// k_gemm_fp4.cuh -- the 4-bit backbone GEMM with the low-rank branches fused
// into its epilogue (FourTune page, section 3.1 Eq. 2 and section 3.2 Eq. 3;
// section 3.3 "LoRA Fusion": the up-projections are fused with the 4-bit
// backbone so the branch outputs accumulate once and Y is written once).
//
//   out[m, n] = ga * gb * sum_k Q(A)[m, k] Q(B)[n, k]
//             + sum_j P[m, j] L1[n, j]            (j < r1)
//             + sum_j P[m, r1 + j] L2[n, j]        (j < r2)
//
// Forward : A = Q(X) [M, K] 1x16,  B = Q(W_res) codes packed along K,
//           P = [X U | s X A], L1 = V, L2 = B.
// Dgrad   : A = Q(dY) [M, N] 1x16, B = Q(W_res)^T codes packed along N with
//           the 16x16 scale grid read transposed (section 3.2: the scale of a
//           16x16 block is the same for W and W^T), P = [dY V | s dY B],
//           L1 = U, L2 = A.
//
// Blackwell mapping: one CTA per SM, persistent over 128x128 output tiles.
//   warp 0  TMA producer: FP4 code tiles (128 B swizzle), raw scale rows,
//           the tile's P / L1 / L2 panels.
//   warp 1  TMEM owner and UMMA issuer: per stage one tcgen05.cp of each
//           operand's block scales into TMEM and four
//           tcgen05.mma.kind::mxf4nvf4.block16 (K = 64 each) into a
//           double-buffered FP32 accumulator, then tcgen05.mma kind::f16 for
//           the low-rank panels into a separate accumulator.  Descriptors
//           are precomputed words, so the issue loop is a few integer adds.
//   warp 2  scale-factor warp: rearranges each stage's scale bytes into the
//           slab layout below, expanding 16x16 weight scales to one per row.
//   warps 4-7 epilogue: tcgen05.ld both accumulators, combine, store.
// TMEM columns: [0,128) acc0, [128,256) acc1, [256,384) low-rank acc,
// [384,400) A scales, [400,416) B scales.
//
// Scale factors in TMEM: the MMA reads the four scale bytes of row m (one
// per 16 K-elements of its K = 64) from TMEM lane m at column c + m/32, c
// being the (4-column aligned) scale address the instruction names.  Each
// K-step's scales are one 32-row x 16-byte slab in shared memory (row m % 32
// holds rows m % 32 + 32 q at bytes 4q..4q+3) that tcgen05.cp.32x128b.warpx4
// replicates into all four lane quarters; K-step j uses columns c = base + 4j.
#pragma once

#include <cuda.h>

#include "ft_ptx.cuh"

namespace ft {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK_BYTES = 128;  // 256 FP4 elements of K per stage
constexpr int KSTEPS = 4;      // MMAs of K = 64 per stage
constexpr int MAX_STAGES = 4;
constexpr int NUM_THREADS = 256;
constexpr int TILE_BYTES = BM * BK_BYTES;      // 16 KiB, A or B stage
constexpr int SFA_RAW_BYTES = BM * 16;         // 128 rows x 16 scale bytes
constexpr int SFB_RAW_BYTES = 256;             // 8 x 16 (fwd) or 16 x 16 (dgrad)
constexpr int SF_ATOM_BYTES = KSTEPS * 512;    // 4 x (32 rows x 16 B)
constexpr int PANEL_BYTES = 128 * 64 * 2;      // a 128-row x 64-col bf16 panel
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL0 = 0, LR_COL = 256, SFA_COL = 384, SFB_COL = 400;

struct Params {
    CUtensorMap mapA, mapB, mapSFA, mapSFB, mapP, mapL1, mapL2;
    const float* ga;
    const float* gb;
    void* out;
    int out_f32;
    int M, Nout, Kc;
    int r1, r2;
    int sfb_trans;
    int stages;
};

struct Layout {
    uint32_t a, b, p, l1, l2, sfa_raw, sfb_raw, sfa, sfb, bars, total;
    int np, n1, n2;
};

__host__ __device__ inline Layout make_layout(int stages, int r1, int r2) {
    Layout L;
    int r = r1 + r2;
    L.np = (r + 63) / 64;
    L.n1 = (r1 + 63) / 64;
    L.n2 = (r2 + 63) / 64;
    uint32_t o = 0;
    L.a = o;        o += stages * TILE_BYTES;
    L.b = o;        o += stages * TILE_BYTES;
    L.p = o;        o += L.np * PANEL_BYTES;
    L.l1 = o;       o += L.n1 * PANEL_BYTES;
    L.l2 = o;       o += L.n2 * PANEL_BYTES;
    L.sfa = o;      o += stages * SF_ATOM_BYTES;
    L.sfb = o;      o += stages * SF_ATOM_BYTES;
    L.sfa_raw = o;  o += stages * SFA_RAW_BYTES;
    L.sfb_raw = o;  o += stages * SFB_RAW_BYTES;
    L.bars = o;     o += 256;  // barriers, TMEM slot, abort flag
    L.total = o + 1024;        // slack for 1 KiB alignment of the base
    return L;
}

// barrier slots (uint64 each) inside the 256-byte barrier area
enum {
    B_FULL = 0,                 // [MAX_STAGES] TMA landed
    B_SF = B_FULL + MAX_STAGES,  // [MAX_STAGES] scale atoms ready
    B_EMPTY = B_SF + MAX_STAGES, // [MAX_STAGES] stage consumed by the MMAs
    B_ACC_FULL = B_EMPTY + MAX_STAGES,  // [2]
    B_ACC_EMPTY = B_ACC_FULL + 2,       // [2]
    B_LR_FULL = B_ACC_EMPTY + 2,
    B_LR_SMEM_EMPTY,
    B_LR_ACC_EMPTY,
    B_DRAIN,
    B_COUNT
};

__global__ void __launch_bounds__(NUM_THREADS, 1) k_gemm_fp4(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const Layout L = make_layout(p.stages, p.r1, p.r2);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.bars + B_COUNT * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.bars + B_COUNT * 8 + 4);

    const int warp = warp_id(), lane = lane_id();
    const int S = p.stages;
    const int r = p.r1 + p.r2;
    const int tiles_m = (p.M + BM - 1) / BM;
    const int tiles_n = p.Nout / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int KT = (p.Kc + 255) / 256;

    if (threadIdx.x == 0) {
        for (int i = 0; i < MAX_STAGES; ++i) {
            mbar_init(&bars[B_FULL + i], 1);
            mbar_init(&bars[B_SF + i], 1);
            mbar_init(&bars[B_EMPTY + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[B_ACC_FULL + i], 1);
            mbar_init(&bars[B_ACC_EMPTY + i], 4);
        }
        mbar_init(&bars[B_LR_FULL], 1);
        mbar_init(&bars[B_LR_SMEM_EMPTY], 1);
        mbar_init(&bars[B_LR_ACC_EMPTY], 4);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.mapA);
        tma_prefetch_desc(&p.mapB);
        tma_prefetch_desc(&p.mapSFA);
        tma_prefetch_desc(&p.mapSFB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint32_t stage_bytes =
                2 * TILE_BYTES + SFA_RAW_BYTES + (p.sfb_trans ? 256u : 128u);
            const uint32_t lr_bytes = (uint32_t)(L.np + L.n1 + L.n2) * PANEL_BYTES;
            uint32_t it = 0;
            bool ok = true;
            int local = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                const int m0 = (tile / tiles_n) * BM;
                const int n0 = (tile % tiles_n) * BN;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait(&bars[B_EMPTY + s], ph ^ 1, ERR_WAIT_EMPTY, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint64_t* fb = &bars[B_FULL + s];
                    mbar_arrive_expect_tx(fb, stage_bytes);
                    tma_load_2d(smem + L.a + s * TILE_BYTES, &p.mapA, fb, kt * BK_BYTES, m0);
                    tma_load_2d(smem + L.b + s * TILE_BYTES, &p.mapB, fb, kt * BK_BYTES, n0);
                    tma_load_2d(smem + L.sfa_raw + s * SFA_RAW_BYTES, &p.mapSFA, fb, kt * 16, m0);
                    if (!p.sfb_trans)
                        tma_load_2d(smem + L.sfb_raw + s * SFB_RAW_BYTES, &p.mapSFB, fb, kt * 16,
                                    n0 / 16);
                    else
                        tma_load_2d(smem + L.sfb_raw + s * SFB_RAW_BYTES, &p.mapSFB, fb,
                                    (n0 / 16) & ~15, kt * 16);
                }
                if (!ok || r == 0) continue;
                // low-rank panels of this tile, after its mainloop loads
                if (!mbar_wait(&bars[B_LR_SMEM_EMPTY], (local & 1) ^ 1, ERR_WAIT_LR, abort_flag)) {
                    ok = false;
                    break;
                }
                uint64_t* lb = &bars[B_LR_FULL];
                mbar_arrive_expect_tx(lb, lr_bytes);
                for (int c = 0; c < L.np; ++c)
                    tma_load_2d(smem + L.p + c * PANEL_BYTES, &p.mapP, lb, c * 64, m0);
                for (int c = 0; c < L.n1; ++c)
                    tma_load_2d(smem + L.l1 + c * PANEL_BYTES, &p.mapL1, lb, c * 64, n0);
                for (int c = 0; c < L.n2; ++c)
                    tma_load_2d(smem + L.l2 + c * PANEL_BYTES, &p.mapL2, lb, c * 64, n0);
            }
            if (!ok) {
                // let copies already issued land before the CTA exits
                for (int d = 0; d < S && d < (int)it; ++d) {
                    uint32_t j = it - 1 - d;
                    volatile int no_abort = 0;
                    mbar_wait(&bars[B_FULL + (j % S)], (j / S) & 1, ERR_WAIT_DRAIN, &no_abort);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_nvfp4(BM, BN);
            const uint32_t idesc_lr = idesc_bf16(BM, BN, 0, 0);
            // descriptor words: lo = start >> 4 | (LBO >> 4) << 16;
            // hi = SBO >> 4 | version 1 << 14 | layout << 29
            const uint32_t hi_sw128 = (1024u >> 4) | (1u << 14) | (SWZ_128B << 29);
            const uint32_t hi_sf = (128u >> 4) | (1u << 14);  // 8-row groups 128 B apart
            const uint32_t a_lo0 = ((base + L.a) >> 4) | (1u << 16);
            const uint32_t b_lo0 = ((base + L.b) >> 4) | (1u << 16);
            const uint32_t sfa_lo0 = (base + L.sfa) >> 4;  // one 16-byte column: LBO unused
            const uint32_t sfb_lo0 = (base + L.sfb) >> 4;
            uint32_t it = 0;
            bool ok = true;
            int local = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                const int b = local & 1;
                const uint32_t acc = tmem + ACC_COL0 + b * BN;
                if (!mbar_wait(&bars[B_ACC_EMPTY + b], ((local >> 1) & 1) ^ 1, ERR_WAIT_ACC_EMPTY,
                               abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait(&bars[B_SF + s], ph, ERR_WAIT_SF, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfa_lo = sfa_lo0 + s * (SF_ATOM_BYTES >> 4);
                    const uint32_t sfb_lo = sfb_lo0 + s * (SF_ATOM_BYTES >> 4);
#pragma unroll
                    for (int j = 0; j < KSTEPS; ++j) {
                        tc_cp_32x128b_x4(tmem + SFA_COL + 4 * j, make_desc(sfa_lo + 32 * j, hi_sf));
                        tc_cp_32x128b_x4(tmem + SFB_COL + 4 * j, make_desc(sfb_lo + 32 * j, hi_sf));
                    }
                    const uint32_t a_lo = a_lo0 + s * (TILE_BYTES >> 4);
                    const uint32_t b_lo = b_lo0 + s * (TILE_BYTES >> 4);
#pragma unroll
                    for (int j = 0; j < KSTEPS; ++j)
                        umma_nvfp4(acc, make_desc(a_lo + 2 * j, hi_sw128), make_desc(b_lo + 2 * j, hi_sw128),
                                   idesc, tmem + SFA_COL + 4 * j, tmem + SFB_COL + 4 * j, (kt | j) != 0);
                    tc_commit(&bars[B_EMPTY + s]);
                }
                if (!ok) break;
                if (r > 0) {
                    if (!mbar_wait(&bars[B_LR_FULL], local & 1, ERR_WAIT_LR, abort_flag) ||
                        !mbar_wait(&bars[B_LR_ACC_EMPTY], (local & 1) ^ 1, ERR_WAIT_LR, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t pP = base + L.p, pL1 = base + L.l1, pL2 = base + L.l2;
                    int q = 0;
                    for (int j = 0; j < p.r1; j += 16, ++q) {
                        uint32_t pa = pP + (j >> 6) * PANEL_BYTES + (j & 63) * 2;
                        uint32_t pb = pL1 + (j >> 6) * PANEL_BYTES + (j & 63) * 2;
                        umma_bf16(tmem + LR_COL, desc_kmajor_sw128(pa), desc_kmajor_sw128(pb), idesc_lr,
                                  q != 0);
                    }
                    for (int j = 0; j < p.r2; j += 16, ++q) {
                        int jp = p.r1 + j;
                        uint32_t pa = pP + (jp >> 6) * PANEL_BYTES + (jp & 63) * 2;
                        uint32_t pb = pL2 + (j >> 6) * PANEL_BYTES + (j & 63) * 2;
                        umma_bf16(tmem + LR_COL, desc_kmajor_sw128(pa), desc_kmajor_sw128(pb), idesc_lr,
                                  q != 0);
                    }
                    tc_commit(&bars[B_LR_SMEM_EMPTY]);
                }
                tc_commit(&bars[B_ACC_FULL + b]);
            }
            // every tcgen05 op issued by this thread completes before TMEM is freed
            tc_commit(&bars[B_DRAIN]);
            volatile int no_abort = 0;
            mbar_wait(&bars[B_DRAIN], 0, ERR_WAIT_DRAIN, &no_abort);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------ scale-factor warp
        uint32_t it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int n0 = (tile % tiles_n) * BN;
            for (int kt = 0; kt < KT; ++kt, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                if (!mbar_wait(&bars[B_FULL + s], ph, ERR_WAIT_FULL, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t raw_a = base + L.sfa_raw + s * SFA_RAW_BYTES;
                const uint32_t raw_b = base + L.sfb_raw + s * SFB_RAW_BYTES;
                const uint32_t at_a = base + L.sfa + s * SF_ATOM_BYTES;
                const uint32_t at_b = base + L.sfb + s * SF_ATOM_BYTES;
                // Rows handled by this lane: m = lane + 32 i (i = 0..3, so m / 32 = i).
                // wa[i][j] / wb[i][j]: the scale word of row m for K-step j.
                uint32_t wa[4][4], wb[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 v = ld_shared_v4(raw_a + (lane + 32 * i) * 16);
                    wa[i][0] = v.x; wa[i][1] = v.y; wa[i][2] = v.z; wa[i][3] = v.w;
                }
                if (!p.sfb_trans) {
                    // raw row y (16 bytes) = scales of rows n0+16y .. +15, 16 K-blocks
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 g = ld_shared_v4(raw_b + ((lane >> 4) + 2 * i) * 16);
                        wb[i][0] = g.x; wb[i][1] = g.y; wb[i][2] = g.z; wb[i][3] = g.w;
                    }
                } else {
                    // raw[y][x]: y = contraction block (16 per stage), x = output
                    // row block starting at (n0/16) & ~15
                    const int xo = (n0 / 16) & 15;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int col = xo + (lane >> 4) + 2 * i;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint32_t v = 0;
#pragma unroll
                            for (int kb = 0; kb < 4; ++kb) {
                                uint32_t byte;
                                asm volatile("ld.shared.u8 %0, [%1];"
                                             : "=r"(byte)
                                             : "r"(raw_b + (4 * j + kb) * 16 + col));
                                v |= (byte & 0xFFu) << (8 * kb);
                            }
                            wb[i][j] = v;
                        }
                    }
                }
                // slab j (512 B) = K-step j: row (lane) at lane * 16 holds the
                // words of rows lane + 32 i, i = 0..3
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(at_a + 512 * j + lane * 16),
                                 "r"(wa[0][j]), "r"(wa[1][j]), "r"(wa[2][j]), "r"(wa[3][j]) : "memory");
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(at_b + 512 * j + lane * 16),
                                 "r"(wb[0][j]), "r"(wb[1][j]), "r"(wb[2][j]), "r"(wb[3][j]) : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_SF + s]);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ epilogue
        const int sp = warp & 3;  // TMEM sub-partition = rows 32*sp .. +31
        bool ok = true;
        int local = 0;
        const float gab = __fmul_rn(*p.ga, *p.gb);
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
            const int b = local & 1;
            const int m0 = (tile / tiles_n) * BM;
            const int n0 = (tile % tiles_n) * BN;
            if (!mbar_wait(&bars[B_ACC_FULL + b], (local >> 1) & 1, ERR_WAIT_ACC_FULL, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int row = m0 + 32 * sp + lane;
            const uint32_t lane_addr = (uint32_t)(32 * sp) << 16;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32], lr[32];
                tmem_ld_32x32b_x32(tmem + lane_addr + ACC_COL0 + b * BN + 32 * c, v);
                if (r > 0) tmem_ld_32x32b_x32(tmem + lane_addr + LR_COL + 32 * c, lr);
                tmem_ld_wait();
                float y[32];
#pragma unroll
                for (int k = 0; k < 32; ++k)
                    y[k] = __fmaf_rn(gab, __uint_as_float(v[k]), r > 0 ? __uint_as_float(lr[k]) : 0.0f);
                if (row < p.M) {
                    if (p.out_f32) {
                        float* o = reinterpret_cast<float*>(p.out) + (int64_t)row * p.Nout + n0 + 32 * c;
#pragma unroll
                        for (int k = 0; k < 32; k += 4)
                            *reinterpret_cast<float4*>(o + k) = make_float4(y[k], y[k + 1], y[k + 2], y[k + 3]);
                    } else {
                        __nv_bfloat16* o =
                            reinterpret_cast<__nv_bfloat16*>(p.out) + (int64_t)row * p.Nout + n0 + 32 * c;
#pragma unroll
                        for (int k = 0; k < 32; k += 8) {
                            uint4 u;
                            __nv_bfloat162 t0 = __floats2bfloat162_rn(y[k], y[k + 1]);
                            __nv_bfloat162 t1 = __floats2bfloat162_rn(y[k + 2], y[k + 3]);
                            __nv_bfloat162 t2 = __floats2bfloat162_rn(y[k + 4], y[k + 5]);
                            __nv_bfloat162 t3 = __floats2bfloat162_rn(y[k + 6], y[k + 7]);
                            u.x = *reinterpret_cast<uint32_t*>(&t0);
                            u.y = *reinterpret_cast<uint32_t*>(&t1);
                            u.z = *reinterpret_cast<uint32_t*>(&t2);
                            u.w = *reinterpret_cast<uint32_t*>(&t3);
                            *reinterpret_cast<uint4*>(o + k) = u;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_ACC_EMPTY + b]);
                if (r > 0) mbar_arrive(&bars[B_LR_ACC_EMPTY]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace gemm
}  // namespace ft
