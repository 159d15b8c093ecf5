// k_qres.cuh -- single-pass LoRA fusion, down side, for inputs that fit in
// the GPU's shared memory (FourTune page, section 3.3: the three branches
// share the input, so quantization and the down-projections read it once).
//
// The NVFP4 tensor scale needs max|T| over the whole input before any code
// can be formed.  A B200 holds 148 x 227 KB of shared memory, more than an
// attention-sized activation ([4608, 3072] bf16 = 28.3 MB), so each CTA
// loads its [128, <= 768] chunk of T once and keeps it resident:
//
//   phase 1  TMA lands the chunk (all of it in flight at once); the
//            quantizer warps take every 1x16 block's max|x| as its stage
//            lands; meanwhile the MMA warp runs the down-projection
//            D[j, m] = sum_c L[c, j] T[m, c] on tcgen05 (kind::f16) over the
//            same tiles, with the factor tiles streamed through a small ring.
//   barrier  the CTA's max is folded into one global word (integer atomicMax
//            on the float bits: exact, order-free); a grid-wide arrival
//            counter (cooperative launch: every CTA is resident) releases all
//            CTAs once every max is in.  Skipped when the caller supplies the
//            tensor amax.
//   phase 2  the tensor scale, the per-scale divisor table, then every block
//            is encoded from shared memory with the block maxima kept in
//            registers since phase 1.
//   tail     TMEM -> FP32 split partials; the last CTA of a row tile adds the
//            splits in split order and rounds P = [bf16(T L1) | bf16(s T L2)].
//
// The arithmetic of every code, scale and P entry is the one of k_qdown and
// k_amax_bf16 (same encoder, same reduction order), so results are
// bit-identical to the two-pass path.
//
// CTA = 128 rows x one C-range of at most 768 columns (12 stages of 64);
// warps: 0 TMA producer, 1 TMEM owner + UMMA issuer, 2-17 quantizers (thread
// t owns row t % 128 and block t / 128 of every 64-column stage) and then
// the epilogue.
#pragma once

#include <cuda.h>

#include "ft_nvfp4.cuh"

namespace ft {
namespace qres {

constexpr int BM = 128;
constexpr int BKC = 64;          // columns per stage (128 bytes of bf16)
constexpr int MAX_ST = 12;       // resident stages per CTA (768 columns)
constexpr int FSTAGES = 2;       // factor-tile ring
constexpr int NQ_WARPS = 16;
constexpr int NQ_THREADS = NQ_WARPS * 32;
constexpr int NUM_THREADS = 64 + NQ_THREADS;
constexpr int TILE_BYTES = BM * BKC * 2;  // 16 KiB
constexpr uint32_t TMEM_COLS = 128;

struct Params {
    CUtensorMap mapT;   // bf16 [M, C], box {64, 128}, 128 B swizzle
    CUtensorMap mapL1;  // direct: L1 [C, r1], box {64, 64}; packed: Lt [128, C], box {64, 128}
    CUtensorMap mapL2;  // direct: L2 [C, r2], box {64, 64}
    const float* amax_in;      // caller's tensor amax, or null (computed here)
    unsigned int* amax_bits;   // global max word, zero on entry (amax_in == null)
    unsigned int* arrivals;    // grid barrier counter, zero on entry (amax_in == null)
    float* tscale;
    uint8_t* codes;
    uint8_t* scales;
    float* part;               // [splits, M, r] FP32 partial down-projections
    __nv_bfloat16* P;          // [M, r]
    unsigned int* counters;    // [row tiles], zero on entry; left zero on exit
    int M, C, r, r1, cchunk, splits;
    float s;
    int do_mma;
    int direct;
    unsigned int num_ctas;
};

struct Layout {
    uint32_t x, f, tab, bars, total;
};

__host__ __device__ inline Layout make_layout(int nst, int do_mma) {
    Layout L;
    uint32_t o = 0;
    L.x = o;    o += (uint32_t)nst * TILE_BYTES;
    L.f = o;    o += do_mma ? (uint32_t)FSTAGES * TILE_BYTES : 0u;
    L.tab = o;  o += (uint32_t)sizeof(QTable);
    L.bars = o; o += 256;
    L.total = o + 1024;  // slack for the 1 KiB alignment of the base
    return L;
}

// barrier slots (uint64 each)
enum {
    QB_XFULL = 0,                    // [MAX_ST] chunk stage landed (used once)
    QB_FFULL = QB_XFULL + MAX_ST,    // [FSTAGES] factor tile landed
    QB_FEMPTY = QB_FFULL + FSTAGES,  // [FSTAGES] factor tile consumed by the MMAs
    QB_ACC = QB_FEMPTY + FSTAGES,    // accumulator complete
    QB_DRAIN,                        // every tcgen05 op of the MMA warp done
    QB_COUNT
};
static_assert(QB_COUNT * 8 + 16 + 4 * NQ_WARPS + 16 <= 256, "barrier area");

// Waits for a phase that must complete (copies already issued) before the
// CTA may exit; bounded like every other wait.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    volatile int no_abort = 0;
    mbar_wait(bar, parity, ERR_WAIT_DRAIN, &no_abort);
}

__global__ void __launch_bounds__(NUM_THREADS, 1) k_qres(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const Layout L = make_layout(p.cchunk / BKC, p.do_mma);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.bars + QB_COUNT * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;
    volatile uint32_t* amax_share = reinterpret_cast<volatile uint32_t*>(last_flag + 1);
    volatile uint32_t* red = amax_share + 1;  // [NQ_WARPS]
    QTable& tab = *reinterpret_cast<QTable*>(smem + L.tab);

    const int warp = warp_id(), lane = lane_id();
    const int m0 = blockIdx.x * BM;
    const int split = blockIdx.y;
    const int c0 = split * p.cchunk;
    const int nst = min(p.cchunk, p.C - c0) / BKC;  // 1 .. MAX_ST

    if (threadIdx.x == 0) {
        for (int i = 0; i < MAX_ST; ++i) mbar_init(&bars[QB_XFULL + i], 1);
        for (int i = 0; i < FSTAGES; ++i) {
            mbar_init(&bars[QB_FFULL + i], 1);
            mbar_init(&bars[QB_FEMPTY + i], 1);
        }
        mbar_init(&bars[QB_ACC], 1);
        mbar_init(&bars[QB_DRAIN], 1);
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
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            // the whole chunk at once: it stays resident
            for (int st = 0; st < nst; ++st) {
                mbar_arrive_expect_tx(&bars[QB_XFULL + st], TILE_BYTES);
                tma_load_2d(smem + L.x + st * TILE_BYTES, &p.mapT, &bars[QB_XFULL + st], c0 + st * BKC, m0);
            }
            int st = 0;
            if (p.do_mma) {
                const int r2 = p.r - p.r1;
                const uint32_t fbytes =
                    !p.direct ? (uint32_t)TILE_BYTES
                              : (p.r1 > 0 ? TILE_BYTES / 2u : 0u) + (r2 > 0 ? TILE_BYTES / 2u : 0u);
                for (; st < nst; ++st) {
                    const int f = st % FSTAGES;
                    const uint32_t ph = (st / FSTAGES) & 1;
                    if (!mbar_wait(&bars[QB_FEMPTY + f], ph ^ 1, ERR_WAIT_EMPTY, abort_flag)) break;
                    uint64_t* fb = &bars[QB_FFULL + f];
                    mbar_arrive_expect_tx(fb, fbytes);
                    uint8_t* dst = smem + L.f + f * TILE_BYTES;
                    const int c = c0 + st * BKC;
                    if (p.direct) {
                        // rank columns 0..63 of rows c .. c+63 of L1 and L2
                        if (p.r1 > 0) tma_load_2d(dst, &p.mapL1, fb, 0, c);
                        if (r2 > 0) tma_load_2d(dst + TILE_BYTES / 2, &p.mapL2, fb, 0, c);
                    } else {
                        tma_load_2d(dst, &p.mapL1, fb, c, 0);
                    }
                }
            }
            if (*abort_flag) {
                // every copy issued lands before the CTA may exit
                for (int s2 = 0; s2 < nst; ++s2) drain_wait(&bars[QB_XFULL + s2], 0);
                for (int d = 0; d < FSTAGES && d < st; ++d) {
                    const int j = st - 1 - d;
                    drain_wait(&bars[QB_FFULL + j % FSTAGES], (j / FSTAGES) & 1);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer
        if (lane == 0 && p.do_mma) {
            // direct: A = [L1 | L2]^T, MN-major (two 64-wide atoms 8 KiB apart,
            // K step = 16 rows = 2 KiB); packed: A = Lt, K-major.  B = T tile.
            const uint32_t idesc = idesc_bf16(128, BM, p.direct ? 1 : 0, 0);
            bool ok = true;
            for (int st = 0; st < nst; ++st) {
                const int f = st % FSTAGES;
                const uint32_t ph = (st / FSTAGES) & 1;
                if (!mbar_wait(&bars[QB_XFULL + st], 0, ERR_WAIT_FULL, abort_flag) ||
                    !mbar_wait(&bars[QB_FFULL + f], ph, ERR_WAIT_FULL, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a = base + L.f + f * TILE_BYTES;
                const uint32_t b = base + L.x + st * TILE_BYTES;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t ad = p.direct ? smem_desc(a + 2048 * j, TILE_BYTES / 2, 1024, SWZ_128B)
                                                 : desc_kmajor_sw128(a + 32 * j);
                    umma_bf16(tmem, ad, desc_kmajor_sw128(b + 32 * j), idesc, (st | j) != 0);
                }
                tc_commit(&bars[QB_FEMPTY + f]);
            }
            if (ok) tc_commit(&bars[QB_ACC]);
            tc_commit(&bars[QB_DRAIN]);
            drain_wait(&bars[QB_DRAIN], 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ quantizers
        const int t = threadIdx.x - 64;
        const int trow = t & (BM - 1), blk = t >> 7;
        const int row = m0 + trow;
        const uint32_t sw = (uint32_t)(trow & 7);
        const uint32_t off_lo = (uint32_t)trow * 128u + (((uint32_t)(2 * blk) ^ sw) << 4);
        const uint32_t off_hi = (uint32_t)trow * 128u + (((uint32_t)(2 * blk + 1) ^ sw) << 4);
        bool ok = true;

        // phase 1: block maxima as the stages land (kept for phase 2)
        uint32_t mb[MAX_ST];
        uint32_t cmax = 0;
#pragma unroll
        for (int st = 0; st < MAX_ST; ++st) {
            mb[st] = 0;
            if (st < nst && ok) {
                if (!mbar_wait(&bars[QB_XFULL + st], 0, ERR_WAIT_FULL, abort_flag)) {
                    ok = false;
                } else {
                    const uint32_t ta = base + L.x + st * TILE_BYTES;
                    const uint4 v0 = ld_shared_v4(ta + off_lo), v1 = ld_shared_v4(ta + off_hi);
                    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                    mb[st] = amax_bits_16(w);
                    cmax = max(cmax, mb[st]);
                }
            }
        }

        // tensor amax: CTA max, then the grid-wide max (or the caller's value)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cmax = max(cmax, __shfl_xor_sync(0xFFFFFFFFu, cmax, o));
        if (lane == 0) red[warp - 2] = cmax;
        named_bar_sync(1, NQ_THREADS);
        if (t == 0) {
            float amax_t;
            if (p.amax_in) {
                amax_t = *p.amax_in;
            } else {
                uint32_t m = 0;
                for (int i = 0; i < NQ_WARPS; ++i) m = max(m, red[i]);
                // every CTA arrives, also one that gave up, so no other CTA
                // waits on it
                if (m) atomicMax(p.amax_bits, m);
                __threadfence();
                red_add_release_gpu(p.arrivals, 1u);
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_gpu(p.arrivals) < p.num_ctas) {
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        report_error(ERR_GRID_SYNC);
                        *abort_flag = 1;
                        break;
                    }
                    __nanosleep(100);
                }
                amax_t = __uint_as_float(ld_acquire_gpu(p.amax_bits));
            }
            *amax_share = __float_as_uint(amax_t);
        }
        named_bar_sync(1, NQ_THREADS);
        const QTensorFast qt = make_qtensor_fast(__uint_as_float(*amax_share));
        build_qtable(tab, qt.g, t, NQ_THREADS);
        if (blockIdx.x == 0 && blockIdx.y == 0 && t == 0) *p.tscale = qt.g;
        named_bar_sync(1, NQ_THREADS);
        ok = ok && !*abort_flag;

        // phase 2: encode every block from shared memory
        if (ok) {
#pragma unroll
            for (int st = 0; st < MAX_ST; ++st) {
                if (st < nst) {
                    const uint32_t ta = base + L.x + st * TILE_BYTES;
                    const uint4 v0 = ld_shared_v4(ta + off_lo), v1 = ld_shared_v4(ta + off_hi);
                    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                    uint32_t sbyte;
                    const uint2 q = quant_block16_fast_m(w, mb[st], qt, tab, sbyte);
                    if (row < p.M) {
                        const int col = c0 + st * BKC + 16 * blk;
                        *reinterpret_cast<uint2*>(p.codes + (int64_t)row * (p.C / 2) + col / 2) = q;
                        p.scales[(int64_t)row * (p.C / 16) + col / 16] = (uint8_t)sbyte;
                    }
                }
            }
        }

        // epilogue: TMEM lane = rank index j, column = tile row; the four
        // warps of a lane quarter take 32 tile rows each
        if (p.do_mma && ok) {
            const int sp = warp & 3;
            const int quarter = (warp - 2) >> 2;
            const int r2 = p.r - p.r1;
            int j;      // P column of this TMEM lane (-1: padding lane)
            bool any;   // warp-uniform: does this lane quarter hold any column
            if (p.direct) {
                const int l = 32 * sp + lane;
                j = (l < 64) ? (l < p.r1 ? l : -1) : (l - 64 < r2 ? p.r1 + l - 64 : -1);
                any = (sp < 2) ? (32 * sp < p.r1) : (32 * (sp - 2) < r2);
            } else {
                j = 32 * sp + lane < p.r ? 32 * sp + lane : -1;
                any = 32 * sp < p.r;
            }
            if (mbar_wait(&bars[QB_ACC], 0, ERR_WAIT_ACC_FULL, abort_flag) && any) {
                tc_fence_after();
                uint32_t v[32];
                const int col0 = 32 * quarter;
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * sp) << 16) + col0, v);
                tmem_ld_wait();
                if (j >= 0) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int m = m0 + col0 + k;
                        if (m < p.M) p.part[((int64_t)split * p.M + m) * p.r + j] = __uint_as_float(v[k]);
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
            const bool lora = j >= p.r1;
            const float a0 = lora ? __fmul_rn(acc[u].x, p.s) : acc[u].x;
            const float a1 = lora ? __fmul_rn(acc[u].y, p.s) : acc[u].y;
            const float a2 = lora ? __fmul_rn(acc[u].z, p.s) : acc[u].z;
            const float a3 = lora ? __fmul_rn(acc[u].w, p.s) : acc[u].w;
            __nv_bfloat162 lo = __floats2bfloat162_rn(a0, a1), hi = __floats2bfloat162_rn(a2, a3);
            uint2 o;
            o.x = *reinterpret_cast<uint32_t*>(&lo);
            o.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(p.P + (int64_t)m0 * p.r + 4 * i) = o;
        }
    }
    if (threadIdx.x == 0) p.counters[blockIdx.x] = 0u;
}

}  // namespace qres
}  // namespace ft
