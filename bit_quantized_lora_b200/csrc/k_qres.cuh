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
//            lands; meanwhile the MMA warp runs the down-projections
//            D[m, j] = sum_c T[m, c] L[c, j] on tcgen05 (kind::f16): A = the
//            same swizzled T tiles (K-major), B = [L1 | L2] as they lie in
//            HBM (MN-major), streamed through a ring: one MMA of N = r per
//            K = 16 step.
//   barrier  the CTA's max is folded into one global word (an integer max on
//            the float bits: exact, order-free); a grid-wide arrival counter
//            releases all CTAs once every max is in.  Every CTA is resident
//            at once: the grid never exceeds the CTAs the device holds (one
//            per SM), and the host launches it plainly (its CTAs wait on the
//            device for the previous kernel) or, on request, cooperatively.
//            Skipped when the caller supplies the tensor amax.
//   phase 2  the tensor scale and the per-scale divisor table, then every
//            block is encoded from shared memory with the block maxima kept
//            in registers since phase 1; each warp's codes leave straight
//            from the encode as whole 32-byte sectors (a warp owns 8 rows x
//            the 4 blocks of a stage), the scale bytes are gathered per row
//            in shared memory and leave in 4-byte and slab stores.  With a
//            caller-supplied tensor amax there is no barrier and no phase 1:
//            each stage is encoded as soon as it lands.
//   P        as soon as the accumulator is complete (during the barrier),
//            four helper warps move TMEM (lane = token, column = P column)
//            to FP32 split partials; in the last CTA of a row tile they add
//            the splits in split order and round P = [bf16(T L1) |
//            bf16(s T L2)] while the quantizer warps are still encoding.
//
// Codes and scales follow the encoding of every other quantizer here, bit
// for bit; P follows k_qdown's rounding (FP32 accumulation, one rounding).
//
// CTA = 128 rows x one C-range of at most 768 columns (12 stages of 64);
// warps: 0 TMA producer, 1 TMEM owner + UMMA issuer, 0-3 then the P path
// (one TMEM lane quarter each), 4-19 quantizers (quantizer warp q owns tile
// rows 8q .. 8q + 7, lane l the block l % 4 of row 8q + l / 4 in every
// 64-column stage).
#pragma once

#include <cuda.h>

#include "ft_nvfp4.cuh"

namespace ft {
namespace qres {

constexpr int BM = 128;
constexpr int BKC = 64;          // columns per stage (128 bytes of bf16)
constexpr int MAX_ST = 12;       // resident stages per CTA (768 columns)
constexpr int MAX_FS = 8;        // factor-ring stages
constexpr int MAX_SPLITS = 8;    // C-splits of one row tile
constexpr int NQ_WARPS = 16;
constexpr int NQ_THREADS = NQ_WARPS * 32;
constexpr int NH_WARPS = 4;      // producer, MMA issuer and two more: the P path
constexpr int NH_THREADS = NH_WARPS * 32;
constexpr int NUM_THREADS = NH_THREADS + NQ_THREADS;
constexpr int TILE_BYTES = BM * BKC * 2;  // 16 KiB
constexpr uint32_t TMEM_COLS = 128;
// staged scale bytes per row: MAX_ST words plus one, so that the byte
// stores of 32 consecutive rows fall in 32 different banks
constexpr uint32_t SROW = MAX_ST * 4 + 4;
constexpr uint32_t BAR_BYTES = 512;
constexpr uint32_t SMEM_LIMIT = 227u * 1024u;

// One low-rank factor L [C, rf] in a ring stage: rf / 16 atoms of 16 rank
// columns x 64 rows of c (32-byte rows, 32-byte swizzle, 2 KiB each), one
// 3-D box per stage.  The second factor's atoms follow the first's, so the
// stage is one MN-major B operand [64, r] whose atoms are ATOM_BYTES apart.
struct Factor {
    int rf;          // rank (0: absent)
    uint32_t off;    // byte offset of its atoms inside a ring stage
};
constexpr uint32_t ATOM_BYTES = 64 * 16 * 2;

struct Params {
    CUtensorMap mapT;   // bf16 [M, C], box {64, 128}, 128 B swizzle
    CUtensorMap mapL1;  // bf16 [C, r1] as {16, C, r1 / 16}, box {16, 64, r1 / 16}, 32 B swizzle
    CUtensorMap mapL2;  // bf16 [C, r2] likewise
    const float* amax_in;      // caller's tensor amax, or null (computed here)
    // epoch-tagged words (any earlier content is fine): [0] grid-barrier
    // arrivals, [1] tensor amax as (epoch << 31) | bits, [2] finished CTAs
    unsigned long long* sync;
    unsigned long long epoch;  // this launch's epoch (host-issued, increasing)
    float* tscale;
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* slab;             // null, or the scales again in the GEMM slab layout
    float* part;               // [splits, M, r] FP32 partial down-projections
    __nv_bfloat16* P;          // [M, r]
    unsigned long long* counters;  // [row tiles] epoch-tagged arrivals of the splits
    int count_done;            // count finished CTAs into sync[2]: the next kernel
                               // may wait on it instead of on this grid's end
    int M, C, r, r1, cchunk, splits;
    float s;
    int do_mma;
    Factor f1, f2;
    uint32_t fstage_bytes;     // one ring stage (both factor tiles)
    int fs;                    // ring stages
    uint32_t ring_bytes;
    unsigned int num_ctas;
};

struct Layout {
    uint32_t x, f, sst, tab, bars, total;
};

__host__ __device__ inline Layout make_layout(int nst, uint32_t ring_bytes) {
    Layout L;
    uint32_t o = 0;
    L.x = o;    o += (uint32_t)nst * TILE_BYTES;
    L.f = o;    o += ring_bytes;  // factor ring
    L.sst = o;  o += BM * SROW;   // staged scale bytes
    L.tab = o;  o += (uint32_t)sizeof(QTableM);
    L.bars = o; o += BAR_BYTES;
    L.total = o + 1024;  // slack for the 1 KiB alignment of the base
    return L;
}

// barrier slots (uint64 each)
enum {
    QB_XFULL = 0,                   // [MAX_ST] chunk stage landed (used once)
    QB_FFULL = QB_XFULL + MAX_ST,   // [MAX_FS] factor tiles landed
    QB_FEMPTY = QB_FFULL + MAX_FS,  // [MAX_FS] factor tiles consumed by the MMAs
    QB_ACC = QB_FEMPTY + MAX_FS,    // accumulator complete
    QB_DRAIN,                       // every tcgen05 op of the MMA warp done
    QB_COUNT
};
static_assert(QB_COUNT * 8 + 16 + 4 * NQ_WARPS <= BAR_BYTES, "barrier area");

// Every global write of this CTA is done: count it (release) for a kernel
// that waits on the counter rather than on this grid's completion.
__device__ __forceinline__ void signal_done(const Params& p) {
    __syncthreads();
    if (threadIdx.x == 0 && p.count_done) {
        __threadfence();
        epoch_count_release(&p.sync[2], p.epoch);
    }
}

// Waits for a phase that must complete (copies already issued) before the
// CTA may exit; bounded like every other wait.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    volatile int no_abort = 0;
    mbar_wait(bar, parity, ERR_WAIT_DRAIN, &no_abort);
}

// TMA load of one factor's atoms for rows c .. c+63 (one 3-D box).
__device__ __forceinline__ void load_factor(uint8_t* stage, const Factor& f, const CUtensorMap* map,
                                            uint64_t* bar, int c) {
    tma_load_3d(stage + f.off, map, bar, 0, c, 0);
}

// P rows of one row tile from the splits' FP32 partials, by threads
// tid = 0 .. NH_THREADS - 1: every split's loads of UNR float4s are issued
// before the first add (one L2 round trip per pass instead of one per
// split), then the adds run in split order.
template <int MAXS, int UNR>
__device__ __forceinline__ void reduce_splits(const Params& p, const float4* part4, int64_t stride4, int n4,
                                              int m0, int tid) {
    for (int i0 = tid; i0 < n4; i0 += UNR * NH_THREADS) {
        float4 v[UNR][MAXS];
#pragma unroll
        for (int k = 0; k < MAXS; ++k) {
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int i = i0 + u * NH_THREADS;
                v[u][k] = (k < p.splits && i < n4) ? __ldcg(part4 + k * stride4 + i)
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int i = i0 + u * NH_THREADS;
            if (i >= n4) continue;
            float4 acc = v[u][0];
#pragma unroll
            for (int k = 1; k < MAXS; ++k) {
                if (k < p.splits) {
                    acc.x = __fadd_rn(acc.x, v[u][k].x);
                    acc.y = __fadd_rn(acc.y, v[u][k].y);
                    acc.z = __fadd_rn(acc.z, v[u][k].z);
                    acc.w = __fadd_rn(acc.w, v[u][k].w);
                }
            }
            const int j = (4 * i) % p.r;  // first of the four columns; r1 % 16 == 0
            const bool lora = j >= p.r1;
            const float a0 = lora ? __fmul_rn(acc.x, p.s) : acc.x;
            const float a1 = lora ? __fmul_rn(acc.y, p.s) : acc.y;
            const float a2 = lora ? __fmul_rn(acc.z, p.s) : acc.z;
            const float a3 = lora ? __fmul_rn(acc.w, p.s) : acc.w;
            __nv_bfloat162 lo = __floats2bfloat162_rn(a0, a1), hi = __floats2bfloat162_rn(a2, a3);
            uint2 o;
            o.x = *reinterpret_cast<uint32_t*>(&lo);
            o.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(p.P + (int64_t)m0 * p.r + 4 * i) = o;
        }
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) k_qres(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const Layout L = make_layout(p.cchunk / BKC, p.ring_bytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.bars + QB_COUNT * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;
    volatile uint32_t* amax_share = reinterpret_cast<volatile uint32_t*>(last_flag + 1);
    volatile uint32_t* red = amax_share + 1;  // [NQ_WARPS]
    QTableM& tab = *reinterpret_cast<QTableM*>(smem + L.tab);

    const int warp = warp_id(), lane = lane_id();
    const int m0 = blockIdx.x * BM;
    const int split = blockIdx.y;
    const int c0 = split * p.cchunk;
    const int nst = min(p.cchunk, p.C - c0) / BKC;  // 1 .. MAX_ST
    const int FS = p.fs;

    if (threadIdx.x == 0) {
        for (int i = 0; i < MAX_ST; ++i) mbar_init(&bars[QB_XFULL + i], 1);
        for (int i = 0; i < MAX_FS; ++i) {
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
    // the previous kernel's outputs are complete from here on; the next
    // kernel may start its own setup
    grid_dep_wait();
    grid_dep_launch();

    if (warp < NH_WARPS) {
        if (warp == 0) {
            // ------------------------------------------------ TMA producer
            if (lane == 0) {
                // the first ring stages of factor tiles (small) ahead of the
                // chunk, so the down-projection starts with the first chunk stage
                const int pre = p.do_mma ? min(FS, nst) : 0;
                for (int st = 0; st < pre; ++st) {
                    uint64_t* fb = &bars[QB_FFULL + st];
                    mbar_arrive_expect_tx(fb, p.fstage_bytes);
                    uint8_t* dst = smem + L.f + st * p.fstage_bytes;
                    if (p.f1.rf > 0) load_factor(dst, p.f1, &p.mapL1, fb, c0 + st * BKC);
                    if (p.f2.rf > 0) load_factor(dst, p.f2, &p.mapL2, fb, c0 + st * BKC);
                }
                // the whole chunk at once: it stays resident
                for (int st = 0; st < nst; ++st) {
                    mbar_arrive_expect_tx(&bars[QB_XFULL + st], TILE_BYTES);
                    tma_load_2d(smem + L.x + st * TILE_BYTES, &p.mapT, &bars[QB_XFULL + st], c0 + st * BKC, m0);
                }
                int st = pre;
                if (p.do_mma) {
                    for (; st < nst; ++st) {
                        const int f = st % FS;
                        const uint32_t ph = (st / FS) & 1;
                        if (!mbar_wait(&bars[QB_FEMPTY + f], ph ^ 1, ERR_WAIT_EMPTY, abort_flag)) break;
                        uint64_t* fb = &bars[QB_FFULL + f];
                        mbar_arrive_expect_tx(fb, p.fstage_bytes);
                        uint8_t* dst = smem + L.f + f * p.fstage_bytes;
                        const int c = c0 + st * BKC;
                        if (p.f1.rf > 0) load_factor(dst, p.f1, &p.mapL1, fb, c);
                        if (p.f2.rf > 0) load_factor(dst, p.f2, &p.mapL2, fb, c);
                    }
                }
                if (*abort_flag) {
                    // every copy issued lands before the CTA may exit
                    for (int s2 = 0; s2 < nst; ++s2) drain_wait(&bars[QB_XFULL + s2], 0);
                    for (int d = 0; d < FS && d < st; ++d) {
                        const int j = st - 1 - d;
                        drain_wait(&bars[QB_FFULL + j % FS], (j / FS) & 1);
                    }
                }
            }
        } else if (warp == 1) {
            // ------------------------------------------------ UMMA issuer
            if (lane == 0 && p.do_mma) {
                // D[:, 0 .. r) (+)= T_tile[:, 16 j ..) (K-major, 128-byte
                // swizzle) x [L1 | L2][16 j .., :) (MN-major 16-column atoms,
                // 32-byte swizzle).  Descriptor words built once: lo = start
                // >> 4 | (LBO >> 4) << 16, hi = SBO >> 4 | version 1 << 14 |
                // swizzle << 29; a K step adds 32 bytes (A) or 16 rows (B).
                const uint32_t idesc = idesc_bf16(128, p.r, 0, 1);
                const uint32_t a_hi = (1024u >> 4) | (1u << 14) | (SWZ_128B << 29);
                const uint32_t b_hi = (256u >> 4) | (1u << 14) | (SWZ_32B << 29);
                const uint32_t a_lo0 = ((base + L.x) >> 4) | (1u << 16);
                const uint32_t b_lo0 = ((base + L.f) >> 4) | ((ATOM_BYTES >> 4) << 16);
                bool ok = true;
                for (int st = 0; st < nst; ++st) {
                    const int f = st % FS;
                    const uint32_t ph = (st / FS) & 1;
                    if (!mbar_wait(&bars[QB_XFULL + st], 0, ERR_WAIT_FULL, abort_flag) ||
                        !mbar_wait(&bars[QB_FFULL + f], ph, ERR_WAIT_FULL, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_lo = a_lo0 + (uint32_t)st * (TILE_BYTES >> 4);
                    const uint32_t b_lo = b_lo0 + (uint32_t)f * (p.fstage_bytes >> 4);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_bf16(tmem, make_desc(a_lo + 2 * j, a_hi), make_desc(b_lo + 32 * j, b_hi), idesc,
                                  (st | j) != 0);
                    tc_commit(&bars[QB_FEMPTY + f]);
                }
                if (ok) tc_commit(&bars[QB_ACC]);
                tc_commit(&bars[QB_DRAIN]);
                drain_wait(&bars[QB_DRAIN], 0);
            }
        }
        __syncwarp();

        // ------------------------------------------------ P path
        // Warp w holds TMEM lanes 32w .. 32w + 31 (token rows).  The split
        // partial leaves as soon as the MMAs are done, which is during the
        // grid barrier; the last CTA of the row tile then adds the splits
        // while its quantizer warps encode.
        if (p.do_mma) {
            if (__all_sync(0xFFFFFFFFu, mbar_wait(&bars[QB_ACC], 0, ERR_WAIT_ACC_FULL, abort_flag))) {
                tc_fence_after();
                const int m = m0 + 32 * warp + lane;
                const uint32_t lane_addr = (uint32_t)(32 * warp) << 16;
                for (int c = 0; c < p.r / 16; ++c) {
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(tmem + lane_addr + 16 * c, v);
                    tmem_ld_wait();
                    if (m < p.M) {
                        float4* o = reinterpret_cast<float4*>(p.part + ((int64_t)split * p.M + m) * p.r + 16 * c);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            o[k] = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                               __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
                    }
                }
            }
            __threadfence();
            named_bar_sync(2, NH_THREADS);
            if (threadIdx.x == 0) {
                // the last CTA of the row tile to arrive adds the splits
                int last = 0;
                if (!*abort_flag) {
                    const unsigned long long prev = epoch_count(&p.counters[blockIdx.x], p.epoch);
                    last = (prev == (unsigned long long)(p.splits - 1)) ? 1 : 0;
                }
                *last_flag = last;
            }
            named_bar_sync(2, NH_THREADS);
            if (*last_flag) {
                // P = [bf16(T L1) | bf16(s T L2)], splits added in split order
                __threadfence();
                const int rows = min(BM, p.M - m0);
                const int n4 = rows * p.r / 4;
                const int64_t stride4 = (int64_t)p.M * p.r / 4;
                const float4* part4 = reinterpret_cast<const float4*>(p.part) + (int64_t)m0 * p.r / 4;
                if (p.splits <= 4)
                    reduce_splits<4, 3>(p, part4, stride4, n4, m0, threadIdx.x);
                else
                    reduce_splits<MAX_SPLITS, 2>(p, part4, stride4, n4, m0, threadIdx.x);
            }
        }
    } else {
        // ------------------------------------------------ quantizers
        // Warp q owns tile rows 8q .. 8q + 7; lane l the block l % 4 of row
        // 8q + l / 4 in every 64-column stage.  A warp's 32 blocks of a stage
        // are then 8 rows x 32 contiguous code bytes: its code stores fill
        // whole 32-byte sectors straight from the encode, and its shared
        // loads (two 16-byte chunks a lane, 128-byte swizzle) are free of
        // bank conflicts within each quarter warp.
        const int t = threadIdx.x - NH_THREADS;
        const int qw = t >> 5;
        const int trow = 8 * qw + (lane >> 2), blk = lane & 3;
        const uint32_t sw = (uint32_t)(trow & 7);
        const uint32_t off_lo = (uint32_t)trow * 128u + (((uint32_t)(2 * blk) ^ sw) << 4);
        const uint32_t off_hi = (uint32_t)trow * 128u + (((uint32_t)(2 * blk + 1) ^ sw) << 4);
        const bool row_ok = m0 + trow < p.M;
        uint8_t* crow = p.codes + (int64_t)(m0 + trow) * (p.C / 2) + c0 / 2 + 8 * blk;
        const uint32_t sstage = base + L.sst;
        bool ok = true;

        // phase 1 (tensor amax computed here): block maxima as the stages
        // land, kept in registers for phase 2
        uint32_t mb[MAX_ST];
        float amax_t = 0.0f;
        if (!p.amax_in) {
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
            // CTA max, then the grid-wide max
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) cmax = max(cmax, __shfl_xor_sync(0xFFFFFFFFu, cmax, o));
            if (lane == 0) red[qw] = cmax;
            named_bar_sync(1, NQ_THREADS);
            if (t == 0) {
                uint32_t m = 0;
                for (int i = 0; i < NQ_WARPS; ++i) m = max(m, red[i]);
                // every CTA arrives, also one that gave up, so no other CTA
                // waits on it; the release orders this CTA's max before its
                // arrival
                atomicMax(&p.sync[1], (p.epoch << 31) | m);
                epoch_count_release(&p.sync[0], p.epoch);
                float a_t = 0.0f;
                if (!epoch_wait(&p.sync[0], p.epoch, p.num_ctas)) {
                    report_error(ERR_GRID_SYNC);
                    *abort_flag = 1;
                } else {
                    const unsigned long long a = ld_acquire_gpu_u64(&p.sync[1]);
                    if ((a >> 31) != p.epoch) {
                        // the word held a value no earlier launch writes
                        report_error(ERR_GRID_SYNC);
                        *abort_flag = 1;
                    }
                    a_t = __uint_as_float((uint32_t)(a & 0x7FFFFFFFull));
                }
                *amax_share = __float_as_uint(a_t);
            }
            named_bar_sync(1, NQ_THREADS);
            amax_t = __uint_as_float(*amax_share);
        } else {
            // the caller's tensor amax: the table is built while the chunk
            // is still in flight, and each stage is encoded as it lands
            amax_t = *p.amax_in;
        }
        const QTensorFast qt = make_qtensor_fast(amax_t);
        build_qtable_m1(tab, qt.g, t, NQ_THREADS);
        if (blockIdx.x == 0 && blockIdx.y == 0 && t == 0) *p.tscale = qt.g;
        named_bar_sync(1, NQ_THREADS);
        build_qtable_m2(tab, t, NQ_THREADS);
        named_bar_sync(1, NQ_THREADS);
        build_qtable_m3(tab, t, NQ_THREADS);
        named_bar_sync(1, NQ_THREADS);
        ok = ok && !*abort_flag;

        // phase 2: encode every block; its 8 code bytes leave at once, its
        // scale byte joins the row's word (lanes 4r .. 4r + 3) in the
        // staging array for the scale and slab stores below
        if (ok) {
#pragma unroll
            for (int st = 0; st < MAX_ST; ++st) {
                if (st < nst && ok) {
                    if (p.amax_in && !mbar_wait(&bars[QB_XFULL + st], 0, ERR_WAIT_FULL, abort_flag)) {
                        ok = false;
                    } else {
                        const uint32_t ta = base + L.x + st * TILE_BYTES;
                        const uint4 v0 = ld_shared_v4(ta + off_lo), v1 = ld_shared_v4(ta + off_hi);
                        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                        uint32_t sbyte;
                        const uint2 q = quant_block16_m(w, p.amax_in ? amax_bits_16(w) : mb[st], qt, tab, sbyte);
                        if (row_ok) *reinterpret_cast<uint2*>(crow + 32 * st) = q;
                        uint32_t sv = sbyte << (8 * blk);
                        sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 1);
                        sv |= __shfl_xor_sync(0xFFFFFFFFu, sv, 2);
                        if (blk == 0) st_shared_u32(sstage + (uint32_t)trow * SROW + st * 4, sv);
                    }
                }
            }
        }
        named_bar_sync(1, NQ_THREADS);
        ok = ok && !*abort_flag;

        if (ok) {
            const int ot = t, on = NQ_THREADS;
            const int rows = min(BM, p.M - m0);
            // scales: one 4-byte word per stage of a row
            for (int i = ot; i < rows * nst; i += on) {
                const int r = i / nst, st = i - r * nst;
                const uint32_t v = ld_shared_u32(sstage + (uint32_t)r * SROW + st * 4);
                *reinterpret_cast<uint32_t*>(p.scales + (int64_t)(m0 + r) * (p.C / 16) + c0 / 16 + 4 * st) = v;
            }
            // the GEMM's scale slabs: slab (row tile, K-step c0 / 64 + st),
            // 16-byte row l = the words of tile rows l, 32 + l, 64 + l, 96 + l
            // (rows past M hold zero scales)
            if (p.slab) {
                for (int i = ot; i < nst * 32; i += on) {
                    const int st = i >> 5, l = i & 31;
                    const uint32_t sa = sstage + (uint32_t)l * SROW + st * 4;
                    const uint4 v = make_uint4(ld_shared_u32(sa), ld_shared_u32(sa + 32 * SROW),
                                               ld_shared_u32(sa + 64 * SROW), ld_shared_u32(sa + 96 * SROW));
                    *reinterpret_cast<uint4*>(p.slab + ((int64_t)blockIdx.x * (p.C / 64) + c0 / 64 + st) * 512 +
                                              l * 16) = v;
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
    signal_done(p);
}

}  // namespace qres
}  // namespace ft
