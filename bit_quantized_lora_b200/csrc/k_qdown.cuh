// k_qdown.cuh -- LoRA fusion, down side (FourTune page, section 3.3: all
// three branches share the input, so quantization and the down-projections
// run as one kernel that reads the input once).
//
// For an input T [M, C] (X in the forward, dY in the backward) one pass
// emits
//   Q(T) : 1x16 NVFP4 codes [M, C/2] and scales [M, C/16]
//   P    : [bf16(T L1) | bf16(s T L2)]  [M, r]
// The down-projection runs on tcgen05 (kind::f16, bf16 in, f32 in TMEM) with
// the roles swapped so the rank is the MMA's M:  D[j, m] = sum_c L[c, j]
// T[m, c].  When r1, r2 <= 64 the A operand is read straight from L1 and L2
// as an MN-major operand: TMA boxes of 64 rank columns (zero-filled past
// r1 / r2) form TMEM lanes 0-63 (L1) and 64-127 (L2).  Otherwise a packed,
// transposed copy Lt = [L1 | L2]^T (k_pack_lt, 128 rows) is read K-major.
// C is split across CTAs; each writes an FP32 partial and the last CTA of a
// row tile (completion counter) adds the partials in split order and rounds
// P with all of its loads in flight at once.
//
// CTA = 128 rows of T x one C-range; warps: 0 TMA producer, 1 UMMA issuer,
// 2-17 quantizers (quantizer warp q owns tile rows 8q .. 8q + 7, lane l the
// block l % 4 of row 8q + l / 4 in each 128 x 64 stage, read from the same
// swizzled shared-memory tile the MMA consumes: a warp's codes of a stage
// are 8 rows x 32 contiguous bytes, whole sectors, and its scales one 4-byte
// word per row, in the row-major and the slab layout alike); warps 2-9 then
// move the down-projection from TMEM to the FP32 partial.
#pragma once

#include <cuda.h>

#include "ft_nvfp4.cuh"

namespace ft {
namespace qdown {

constexpr int BM = 128;
constexpr int BKC = 64;  // columns of T per stage (128 bytes of bf16)
constexpr int STAGES = 4;
constexpr int NQ_WARPS = 16;  // quantizer warps (the first 8 also the epilogue)
constexpr int NUM_THREADS = 64 + NQ_WARPS * 32;
constexpr int TILE_BYTES = BM * BKC * 2;  // 16 KiB
constexpr uint32_t TMEM_COLS = 128;

struct Params {
    CUtensorMap mapT;   // bf16 [M, C], box {64, 128}, 128 B swizzle
    CUtensorMap mapL1;  // direct: L1 [C, r1], box {64, 64}; packed: Lt [128, C], box {64, 128}
    CUtensorMap mapL2;  // direct: L2 [C, r2], box {64, 64}
    const float* amax;
    float* tscale;
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* slab;             // the scales again in the GEMM slab layout
    float* part;               // [splits, M, r] FP32 partial down-projections
    __nv_bfloat16* P;          // [M, r] result
    unsigned int* counters;    // [row tiles], zero on entry; left zero on exit
    int M, C, r, r1, cchunk, splits;
    float s;
    int do_mma;
    int direct;  // 1: read L1 / L2 directly (r1, r2 <= 64); 0: packed Lt
    int quant;   // 1: Q(T) and P; 0: P alone (T already quantized elsewhere)
};

constexpr uint32_t SMEM_BYTES = STAGES * 2 * TILE_BYTES + sizeof(QTableM) + 256 + 1024;

__global__ void __launch_bounds__(NUM_THREADS, 1) k_qdown(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const uint32_t off_x = 0, off_l = STAGES * TILE_BYTES, off_tab = 2 * STAGES * TILE_BYTES;
    const uint32_t off_bar = off_tab + sizeof(QTableM);
    QTableM& tab = *reinterpret_cast<QTableM*>(smem + off_tab);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + off_bar);
    uint64_t* empty = full + STAGES;
    uint64_t* accfull = empty + STAGES;
    uint64_t* drain = accfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;

    const int warp = warp_id(), lane = lane_id();
    const int m0 = blockIdx.x * BM;
    const int split = blockIdx.y;
    const int c0 = split * p.cchunk;
    const int cn = min(p.cchunk, p.C - c0);
    const int nst = cn / BKC;
    const QTensorFast qt = make_qtensor_fast(p.quant ? *p.amax : 0.0f);

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            // every quantizer warp releases the stage after its own loads
            // (behind a proxy fence, see below), plus the MMA commit
            mbar_init(&empty[i], (p.quant ? NQ_WARPS : 0) + (p.do_mma ? 1 : 0));
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
            const int r2 = p.r - p.r1;
            const uint32_t bytes =
                TILE_BYTES + (!p.do_mma ? 0u
                              : !p.direct ? (uint32_t)TILE_BYTES
                                          : (p.r1 > 0 ? TILE_BYTES / 2u : 0u) + (r2 > 0 ? TILE_BYTES / 2u : 0u));
            int st = 0;
            for (; st < nst; ++st) {
                const int s = st % STAGES;
                const uint32_t ph = (st / STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, ERR_WAIT_EMPTY, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(smem + off_x + s * TILE_BYTES, &p.mapT, &full[s], c0 + st * BKC, m0);
                if (p.do_mma) {
                    if (p.direct) {
                        // rank columns 0..63 of rows c0 + 64 st .. +63 of L1 and L2
                        // (an absent factor leaves its lanes unused)
                        if (p.r1 > 0)
                            tma_load_2d(smem + off_l + s * TILE_BYTES, &p.mapL1, &full[s], 0, c0 + st * BKC);
                        if (r2 > 0)
                            tma_load_2d(smem + off_l + s * TILE_BYTES + TILE_BYTES / 2, &p.mapL2, &full[s], 0,
                                        c0 + st * BKC);
                    } else {
                        tma_load_2d(smem + off_l + s * TILE_BYTES, &p.mapL1, &full[s], c0 + st * BKC, 0);
                    }
                }
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
            // direct: A = [L1 | L2]^T, MN-major (two 64-wide atoms 8 KiB apart,
            // K step = 16 rows = 2 KiB); packed: A = Lt, K-major
            const uint32_t idesc = idesc_bf16(128, BM, p.direct ? 1 : 0, 0);
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
                for (int j = 0; j < 4; ++j) {
                    const uint64_t ad = p.direct ? smem_desc(a + 2048 * j, TILE_BYTES / 2, 1024, SWZ_128B)
                                                 : desc_kmajor_sw128(a + 32 * j);
                    umma_bf16(tmem, ad, desc_kmajor_sw128(b + 32 * j), idesc, (st | j) != 0);
                }
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(accfull);
            tc_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, ERR_WAIT_DRAIN, &no_abort);
        }
        __syncwarp();
    } else {
        // quantizers
        const int t = threadIdx.x - 64;
        const int qw = t >> 5;
        const int trow = 8 * qw + (lane >> 2), blk = lane & 3;
        const int row = m0 + trow;
        if (p.quant && blockIdx.x == 0 && blockIdx.y == 0 && t == 0) *p.tscale = qt.g;
        // the multiply-path table, built while the first stages land
        build_qtable_m1(tab, qt.g, t, NQ_WARPS * 32);
        named_bar_sync(1, NQ_WARPS * 32);
        build_qtable_m2(tab, t, NQ_WARPS * 32);
        named_bar_sync(1, NQ_WARPS * 32);
        build_qtable_m3(tab, t, NQ_WARPS * 32);
        named_bar_sync(1, NQ_WARPS * 32);
        bool ok = true;
        const uint32_t sw = (uint32_t)(trow & 7);
        const uint32_t off_lo = (uint32_t)trow * 128u + (((uint32_t)(2 * blk) ^ sw) << 4);
        const uint32_t off_hi = (uint32_t)trow * 128u + (((uint32_t)(2 * blk + 1) ^ sw) << 4);
        for (int st = 0; st < (p.quant ? nst : 0); ++st) {
            const int s = st % STAGES;
            const uint32_t ph = (st / STAGES) & 1;
            if (!mbar_wait(&full[s], ph, ERR_WAIT_FULL, abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t ta = base + off_x + s * TILE_BYTES;
            const uint4 v0 = ld_shared_v4(ta + off_lo), v1 = ld_shared_v4(ta + off_hi);
            // the next TMA copy into this stage is an async-proxy write: the
            // generic-proxy loads above must be ordered before it explicitly
            // (without this fence the copy was seen to overtake them)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            uint32_t sbyte;
            const uint2 q = quant_block16_m(w, amax_bits_16(w), qt, tab, sbyte);
            // the row's four scale bytes of this stage (lanes 4r .. 4r + 3)
            uint32_t sv = sbyte << (8 * blk);
            sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 1);
            sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 2);
            if (row < p.M) {
                const int col = c0 + st * BKC;
                *reinterpret_cast<uint2*>(p.codes + (int64_t)row * (p.C / 2) + col / 2 + 8 * blk) = q;
                if (blk == 0) {
                    *reinterpret_cast<uint32_t*>(p.scales + (int64_t)row * (p.C / 16) + col / 16) = sv;
                    *reinterpret_cast<uint32_t*>(p.slab + slab_offset(row, col / 16, p.C)) = sv;
                }
            }
        }
        if (p.do_mma && ok && warp < 10) {
            // TMEM lane = rank index j, column = tile row; warps 2-5 take tile
            // rows 0-63, warps 6-9 rows 64-127
            const int sp = warp & 3;
            const int half = (warp - 2) >> 2;
            const int r2 = p.r - p.r1;
            // TMEM lane -> P column (-1: padding lane)
            int j;
            bool any;  // warp-uniform: does this lane quarter hold any column
            if (p.direct) {
                const int l = 32 * sp + lane;
                j = (l < 64) ? (l < p.r1 ? l : -1) : (l - 64 < r2 ? p.r1 + l - 64 : -1);
                any = (sp < 2) ? (32 * sp < p.r1) : (32 * (sp - 2) < r2);
            } else {
                j = 32 * sp + lane < p.r ? 32 * sp + lane : -1;
                any = 32 * sp < p.r;
            }
            if (mbar_wait(accfull, 0, ERR_WAIT_ACC_FULL, abort_flag) && any) {
                tc_fence_after();
                const uint32_t lane_addr = (uint32_t)(32 * sp) << 16;
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    uint32_t v[32];
                    const int col0 = 64 * half + 32 * c;
                    tmem_ld_32x32b_x32(tmem + lane_addr + col0, v);
                    tmem_ld_wait();
                    if (j >= 0) {
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const int m = m0 + col0 + k;
                            if (m < p.M)
                                p.part[((int64_t)split * p.M + m) * p.r + j] = __uint_as_float(v[k]);
                        }
                    }
                }
            }
        }
    }
    // every thread's partial writes become visible device-wide before the
    // completion counter below is bumped
    __threadfence();
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && p.do_mma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (!p.do_mma || *abort_flag) return;

    // The last CTA of this row tile to finish adds the splits' partials in
    // split order (deterministic) and rounds P = [bf16(T L1) | bf16(s T L2)].
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&p.counters[blockIdx.x], 1u);
        *last_flag = (prev == (unsigned)(p.splits - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (!*last_flag) return;
    __threadfence();
    // all partials of the tile's rows, 4 floats at a time (r % 16 == 0), with
    // every split's load of a batch in flight together
    const int rows = min(BM, p.M - m0);
    const int n4 = rows * p.r / 4;
    const int64_t stride4 = (int64_t)p.M * p.r / 4;
    const float4* part4 = reinterpret_cast<const float4*>(p.part) + (int64_t)m0 * p.r / 4;
    constexpr int UNR = 4;
    for (int i0 = threadIdx.x; i0 < n4; i0 += UNR * NUM_THREADS) {
        float4 acc[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < p.splits; ++k) {
            float4 v[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int i = i0 + u * NUM_THREADS;
                v[u] = i < n4 ? __ldcg(part4 + k * stride4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                acc[u].x = __fadd_rn(acc[u].x, v[u].x);
                acc[u].y = __fadd_rn(acc[u].y, v[u].y);
                acc[u].z = __fadd_rn(acc[u].z, v[u].z);
                acc[u].w = __fadd_rn(acc[u].w, v[u].w);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int i = i0 + u * NUM_THREADS;
            if (i >= n4) continue;
            const int j = (4 * i) % p.r;  // first of the four columns; r1 % 16 == 0
            const float sc = j >= p.r1 ? p.s : 1.0f;
            const float a0 = j >= p.r1 ? __fmul_rn(acc[u].x, sc) : acc[u].x;
            const float a1 = j >= p.r1 ? __fmul_rn(acc[u].y, sc) : acc[u].y;
            const float a2 = j >= p.r1 ? __fmul_rn(acc[u].z, sc) : acc[u].z;
            const float a3 = j >= p.r1 ? __fmul_rn(acc[u].w, sc) : acc[u].w;
            __nv_bfloat162 lo = __floats2bfloat162_rn(a0, a1), hi = __floats2bfloat162_rn(a2, a3);
            uint2 o;
            o.x = *reinterpret_cast<uint32_t*>(&lo);
            o.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(p.P + (int64_t)m0 * p.r + 4 * i) = o;
        }
    }
    if (threadIdx.x == 0) p.counters[blockIdx.x] = 0u;
}

}  // namespace qdown

// Lt[j, c] = L1[c, j] (j < r1), L2[c, j - r1] (j < r1 + r2), 0 (j < 128):
// the transposed, zero-padded low-rank factor the down-projection MMA reads
// when a rank exceeds 64.  Grid (ceil(C / 256), 128): one output row j per
// blockIdx.y, coalesced writes.
__global__ void __launch_bounds__(256) k_pack_lt(const uint16_t* __restrict__ L1, int r1,
                                                 const uint16_t* __restrict__ L2, int r2, int C,
                                                 uint16_t* __restrict__ Lt) {
    const int j = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c >= C) return;
    uint16_t v = 0;
    if (j < r1)
        v = L1[(int64_t)c * r1 + j];
    else if (j < r1 + r2)
        v = L2[(int64_t)c * r2 + (j - r1)];
    Lt[(int64_t)j * C + c] = v;
}

}  // namespace ft
