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
// Dgrad   : A = Q(dY) [M, N] 1x16, B = Q(W_res)^T codes packed along N,
//           P = [dY V | s dY B], L1 = U, L2 = A.
//
// Block scales arrive in the tensor-memory slab layout (below): the
// activation quantizers write it next to the row-major scales; the weight's
// 16x16 grid is expanded into it once per layer, for both code layouts, and
// stored behind each 256 x 256 block of codes in the weight's operand image
// (section 3.2: one grid serves W and W^T; the expansion repeats each 16x16
// scale for its 16 rows and changes no code).
// Slab layout of an operand with R rows and Kc contraction columns:
// [ceil(R/128)][Kc/64][512 B], byte 16 l + 4 i + b of slab (t, s) = the
// scale of row 128 t + 32 i + l, 16-column block 4 s + b.  One slab is
// exactly what tcgen05.cp.32x128b.warpx4 turns into the scale layout the
// MMA reads (row m at TMEM lane m % 32 of every lane quarter, column
// c + m / 32).
//
// Blackwell mapping: one CTA per SM, persistent over 128x256 output tiles
// (a tcgen05 MMA costs about the same for N = 128 as for N = 256, so the
// wide tile doubles the work per instruction); or, the default for more
// than 128 rows, CTA pairs on 256x256 tiles (kPair, below).  The MMA queue
// is shallow: every instruction the MMA thread runs between MMAs costs
// tensor-pipe time, so its per-stage path is kept to one non-suspending
// barrier check, the MMAs and the commits (ring slots advance by increments).
//   warp 0  TMA producer: per stage, the weight block (codes + scales, one
//           3-D box) and the activation scale slabs on one barrier, the
//           activation code tile (128 B swizzle) on another; per tile the
//           P / L1 / L2 panels, issued once the ring holds the tile's first
//           stages (they are read after the tile's mainloop).
//   warp 1  TMEM owner and UMMA issuer: four
//           tcgen05.mma.kind::mxf4nvf4.block16 (K = 64, N = 256) per stage
//           into the FP32 accumulator, then the low-rank up-projection
//           (kind::f16, two halves of N = 128).
//   warps 2-5  scale warps, one per TMEM lane quarter (2, 3, 0, 1): each
//           lane loads its 16-byte slab row of every K step from shared
//           memory and writes it with tcgen05.st into its own lane of a
//           two-deep ring of scale columns -- the replicated contents a
//           tcgen05.cp 32x128b.warpx4 per slab would leave, without the
//           ~52 tensor-pipe cycles each of those twelve copies a stage costs.
//   warps 6-13 epilogue, two groups working on the two column halves at
//           once: tcgen05.ld accumulator and low-rank half into registers
//           (16 columns at a time), release tensor memory, combine, stage
//           and store Y once.
// TMEM columns: [0,256) accumulator, [256,384) low-rank half 0, [384,512)
// the scale ring (per slot: A 16 columns, B 32 columns) during the mainloop
// and low-rank half 1 after it.
//
// Low-rank panels are K-major with the rank as K, each factor's part of P
// and the factor itself swizzled to its own width (16, 32 or 64 columns per
// 32, 64 or 128-byte row; two 64-column atoms above 64).
#pragma once

#include <cuda.h>

#include "ft_gelu.cuh"
#include "ft_nvfp4.cuh"
#include "ft_ptx.cuh"

namespace ft {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK_BYTES = 128;  // 256 FP4 elements of K per stage
constexpr int KSTEPS = 4;      // MMAs of K = 64 per stage
constexpr int MAX_STAGES = 4;
constexpr int NUM_EPI_WARPS = 8;  // two column groups of four lane-quarter warps
constexpr int NUM_SF_WARPS = 4;   // one per TMEM lane quarter
constexpr int EPI_WARP0 = 2 + NUM_SF_WARPS;
constexpr int NUM_THREADS = 32 * (EPI_WARP0 + NUM_EPI_WARPS);
constexpr int A_BYTES = BM * BK_BYTES;         // 16 KiB
constexpr int B_BYTES = BN * BK_BYTES;         // 32 KiB of codes
constexpr int SFA_STAGE_BYTES = KSTEPS * 512;  // four slabs (128 rows)
constexpr int SFB_STAGE_BYTES = 2 * KSTEPS * 512;  // two row halves x four slabs
// one block of the weight's operand image: the B tile's codes, then its
// scale slabs (they arrive in one copy)
constexpr int B_SLOT = B_BYTES + SFB_STAGE_BYTES;  // 36 KiB
// CTA pairs: each CTA holds its 128-row half of the B tile's codes and the
// scale slabs of all 256 rows (its accumulator spans every column)
constexpr int B_HALF_BYTES = (BN / 2) * BK_BYTES;          // 16 KiB
constexpr int B_SLOT_P = B_HALF_BYTES + SFB_STAGE_BYTES;    // 20 KiB
// rows of one 256-row block of the weight's operand image: 256 code rows of
// 128 bytes, then its 32 rows of scale slabs
constexpr int IMG_BLOCK_ROWS = 288;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns: [0,256) accumulator; [256,384) low-rank half 0; [384,512)
// shared in time: the scale ring while the mainloop runs, low-rank half 1
// after it (the next tile's first scale copy waits for the epilogue).
constexpr uint32_t ACC_COL = 0, LR0_COL = 256, R2_COL = 384, SF_SLOT_COLS = 48;
// CTA pairs: each stage slot s keeps its scales in columns
// [256 + 48 s, 256 + 48 s + 48) during the mainloop (at most four stages,
// [256, 448)); both low-rank halves are computed after it, into [256, 512).
// The barrier arrays below are sized for SF_SLOTS_P slots.
constexpr int SF_SLOTS = 2, SF_SLOTS_P = 5;
constexpr uint32_t RING_COL_P = LR0_COL;

// One low-rank factor's panels: P columns [pcol, pcol + rf) for the tile's
// 128 rows (A operand) and L [256 output rows, rf] (B operand), both K-major.
struct LrFactor {
    int rf;        // rank (0: absent)
    int wbox;      // 16, 32 or 64 elements per swizzled row
    int natoms;    // 1, or 2 above 64
    int pcol;      // first column of P
    uint32_t swz;  // descriptor swizzle code
    uint32_t row_bytes;  // wbox x 2
};

struct Params {
    CUtensorMap mapA, mapB, mapP1, mapP2, mapL1, mapL2;
    // the block-scale slabs ([tiles][Kc/64][512 B], activations and weights)
    // as 3-D tensors {256 B, 2 * Kc / 64, tiles}: one stage's four slabs are
    // one box (8 x 256 B) of one tile (A) or of two (B)
    CUtensorMap mapSFA;
    // CTA pairs: mapB covers one CTA's 128 code rows of an image block,
    // mapBs the block's 32 rows of scale slabs; mapL1 / mapL2 boxes are 64
    // rows (one CTA's share of a 128-column half)
    CUtensorMap mapBs;
    const float* ga;
    const float* gb;
    uint8_t* out;        // output [M, Nout], bf16 or FP32, rows contiguous
    const unsigned long long* dep_done;  // null, or the producer's finished-CTA counter,
    unsigned long long dep_epoch;        // its epoch
    unsigned int dep_count;              // and its grid size
    int out_f32;
    int M, Nout, Kc;
    LrFactor f1, f2;
    int stages;
    // MLP fusion (section 3.3; bf16 output only): the output is H =
    // GELU(bf16(y)), and the epilogue also quantizes H for the next linear
    // with the tensor scale of the caller's amax_h: 1x16 codes [M, Nout/2],
    // scales [M, Nout/16], the same scales in the GEMM slab layout, and the
    // decode scale (written by CTA 0)
    int mlp;
    const float* amax_h;
    uint8_t* q_codes;
    uint8_t* q_scales;
    uint8_t* q_slab;
    float* q_tscale;
    // null, or a float (as its bits) raised to the largest |value| the
    // epilogue writes (bf16 Y or H as rounded, FP32 Y as stored): the next
    // quantizer's tensor amax, found without another pass
    unsigned int* amax_out;
};

struct Layout {
    uint32_t a, b, sfa, p1, p2, l1, l2, stg, tab, bars, total;
};
constexpr uint32_t STG_BYTES = 128 * 32;  // one staged output chunk: 128 rows x 32 bytes

// bytes of a factor's P panel (128 rows) and L panel (256 rows; a CTA of a
// pair holds 128 of them)
__host__ __device__ inline uint32_t p_bytes(const LrFactor& f) {
    return f.rf > 0 ? (uint32_t)f.natoms * 128u * f.row_bytes : 0u;
}
__host__ __device__ inline uint32_t l_bytes(const LrFactor& f) {
    return f.rf > 0 ? (uint32_t)f.natoms * 256u * f.row_bytes : 0u;
}

__host__ __device__ inline Layout make_layout(int stages, const LrFactor& f1, const LrFactor& f2, int mlp,
                                              int pair = 0) {
    Layout L;
    uint32_t o = 0;
    const uint32_t lsh = pair ? 1u : 0u;
    L.a = o;    o += stages * A_BYTES;
    L.b = o;    o += stages * (pair ? B_SLOT_P : B_SLOT);
    L.p1 = o;   o += p_bytes(f1);
    L.l1 = o;   o += l_bytes(f1) >> lsh;
    L.p2 = o;   o += p_bytes(f2);
    L.l2 = o;   o += l_bytes(f2) >> lsh;
    L.sfa = o;  o += stages * SFA_STAGE_BYTES;
    L.stg = o;  o += mlp ? 0u : 2 * STG_BYTES;  // output staging, one buffer per column group (H: none)
    L.tab = o;  o += mlp ? (uint32_t)sizeof(QTableM) + 2u * kGeluTab : 0u;  // Q(H)'s encode table, GELU's
    o = (o + 15u) & ~15u;
    L.bars = o; o += 256;  // barriers, TMEM slot, abort flag
    L.total = o + 1024;    // slack for 1 KiB alignment of the base
    return L;
}

// barrier slots (uint64 each) inside the 256-byte barrier area
enum {
    B_FULL = 0,                        // [MAX_STAGES] TMA landed
    B_EMPTY = B_FULL + MAX_STAGES,     // [MAX_STAGES] stage consumed by the MMAs
    B_SFFULL = B_EMPTY + MAX_STAGES,   // [MAX_STAGES] the stage's scale slabs landed
    B_SF_READY = B_SFFULL + MAX_STAGES, // [SF_SLOTS_P] scale slot copied into TMEM
    B_SF_FREE = B_SF_READY + SF_SLOTS_P, // [SF_SLOTS_P] scale slot read by its MMAs
    B_ACC_FULL = B_SF_FREE + SF_SLOTS_P,
    B_ACC_EMPTY,                       // every epilogue warp done with the tile
    B_LR_FULL,                         // panels landed
    B_LR_SMEM_EMPTY,                   // panels consumed
    B_LR0_READY,                       // low-rank half 0 computed
    B_LR1_READY,                       // low-rank half 1 computed
    B_DRAIN,
    B_EPI_DONE,                        // this CTA's epilogue done with the tile (CTA pairs)
    B_COUNT
};
static_assert(B_COUNT * 8 + 8 <= 256, "barrier area");

// The K = 16 MMAs of one factor's up-projection for output columns
// [128 h, 128 h + 128) of the tile: D (+)= P_f x L_f[half h]^T.
// Descriptor words are built once per call (lo = start >> 4 | 1 << 16,
// hi = SBO >> 4 | version 1 << 14 | swizzle << 29); a K step adds 32 bytes
// inside an atom, the second 64-wide atom (rf > 64) starts a panel later.
// kPair: the pair's MMA (M = 256); each CTA's L panel holds its 64 rows of
// each half, so halves are 64 rows apart and atoms 128.
template <bool kPair>
__device__ __forceinline__ void lr_mma(uint32_t tmem_d, uint32_t pa, uint32_t pb, const LrFactor& f, int h,
                                       uint32_t idesc, int& q) {
    constexpr uint32_t HALF = kPair ? 64u : 128u;
    const uint32_t hi = ((8u * f.row_bytes) >> 4) | (1u << 14) | (f.swz << 29);
    const uint32_t a_lo = (pa >> 4) | (1u << 16);
    const uint32_t b_lo = ((pb + (uint32_t)h * HALF * f.row_bytes) >> 4) | (1u << 16);
    const uint32_t a_atom = (128u * f.row_bytes) >> 4, b_atom = (2u * HALF * f.row_bytes) >> 4;
    for (int j = 0; j < f.rf; j += 16, ++q) {
        const uint32_t a = (uint32_t)(j >> 6), k = ((uint32_t)(j & (f.wbox - 1)) * 2u) >> 4;
        if (kPair)
            umma_bf16_pair(tmem_d, make_desc(a_lo + a * a_atom + k, hi), make_desc(b_lo + a * b_atom + k, hi), idesc,
                           q != 0);
        else
            umma_bf16(tmem_d, make_desc(a_lo + a * a_atom + k, hi), make_desc(b_lo + a * b_atom + k, hi), idesc,
                      q != 0);
    }
}

// kBf16 = false: the 4-bit backbone GEMM (both operands NVFP4, block
// scales staged in tensor memory); a 256-deep stage is four K = 64 MMAs.
// kBf16 = true: the 16-bit variant of the precision ablation (FourTune
// page, section 4, Table 4): A = a bf16 activation or gradient, B = the
// weight's bf16 image (E2M1 value x block scale, exact in bf16; the tensor
// scale stays apart as gb), tcgen05 kind::f16; a stage holds 64 columns of
// K in the same 128-byte rows, four K = 16 MMAs.  No scale factors: the
// scale warps idle.  Tiles, epilogue and low-rank terms are shared.
// kMlp: the MLP-fusion epilogue (Params::mlp), for the 4-bit GEMM.
// kPair: the 4-bit GEMM on CTA pairs (clusters of two): 256 x 256 tiles,
// CTA r of a pair owns output rows 128 r .. 128 r + 127 of the tile and
// loads its own A rows, its half of the B codes and all of the tile's
// scales; the leader's MMAs (M = 256) read both CTAs' operands, so each SM
// waits for 38 KB per stage instead of 54 KB for the same work.
template <bool kBf16, bool kMlp = false, bool kPair = false>
__global__ void __launch_bounds__(NUM_THREADS, 1) k_gemm_fp4(const __grid_constant__ Params p) {
    static_assert(!(kBf16 && kPair), "CTA pairs are for the 4-bit GEMM");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const Layout L = make_layout(p.stages, p.f1, p.f2, kMlp ? 1 : 0, kPair ? 1 : 0);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.bars + B_COUNT * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.bars + B_COUNT * 8 + 4);

    const int warp = warp_id(), lane = lane_id();
    const int S = p.stages;
    const bool has_lr = p.f1.rf + p.f2.rf > 0;
    // output rows per tile: the CTA's 128, or the pair's 256 (this CTA's
    // rows start at 128 rank); both CTAs of a pair walk the same tiles
    constexpr int TM = kPair ? 2 * BM : BM;
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;
    const int unit = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int nunits = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int tiles_m = (p.M + TM - 1) / TM;
    const int tiles_n = p.Nout / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int KT = kBf16 ? p.Kc / 64 : p.Kc / 256;  // stages per tile

    if (threadIdx.x == 0) {
        for (int i = 0; i < MAX_STAGES; ++i) {
            // CTA pairs: the leader's FULL also counts both CTAs' scale warps
            // (the stage's scales are in tensor memory), so the MMA thread
            // waits on one barrier per stage
            mbar_init(&bars[B_FULL + i], kPair ? 1 + 2 * NUM_SF_WARPS : 1);
            mbar_init(&bars[B_SFFULL + i], 1);
            mbar_init(&bars[B_EMPTY + i], 1);
        }
        // a pair's leader counts both CTAs' scale and epilogue warps
        for (int i = 0; i < SF_SLOTS_P; ++i) {
            mbar_init(&bars[B_SF_READY + i], (kPair ? 2 : 1) * NUM_SF_WARPS);
            mbar_init(&bars[B_SF_FREE + i], 1);
        }
        mbar_init(&bars[B_ACC_FULL], 1);
        mbar_init(&bars[B_ACC_EMPTY], (kPair ? 2 : 1) * NUM_EPI_WARPS);
        mbar_init(&bars[B_EPI_DONE], NUM_EPI_WARPS);
        mbar_init(&bars[B_LR_FULL], 1);
        mbar_init(&bars[B_LR_SMEM_EMPTY], 1);
        mbar_init(&bars[B_LR0_READY], 1);
        mbar_init(&bars[B_LR1_READY], 1);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.mapA);
        tma_prefetch_desc(&p.mapB);
        if (!kBf16) tma_prefetch_desc(&p.mapSFA);
    }
    // both CTAs' barriers exist before either signals the other's
    if constexpr (kPair) cluster_sync();
    if (warp == 1) {
        if (kPair) {
            tmem_alloc_pair(tmem_slot, TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (kPair) cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the inputs written by the previous kernel are complete from here on;
    // the next kernel may start its own setup
    wait_inputs(p.dep_done, p.dep_epoch, p.dep_count, abort_flag);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (kPair && lane == 0) {
            // Per stage: this CTA's A rows and B code half, with their bytes
            // counted on the leader's FULL barrier (the leader expects both
            // CTAs' bytes); the tile's weight scale slabs (all 256 rows) and
            // this CTA's activation slabs on its own SFFULL barrier, for its
            // scale warps.  Panels likewise: this CTA's 128 rows of P and its
            // 64 rows of each half of L, counted on the leader's LR_FULL.
            const uint32_t lead_full = mapa_shared(smem_u32(&bars[B_FULL]), 0);
            const uint32_t lead_lr = mapa_shared(smem_u32(&bars[B_LR_FULL]), 0);
            const uint32_t lr_share = p_bytes(p.f1) + (l_bytes(p.f1) >> 1) + p_bytes(p.f2) + (l_bytes(p.f2) >> 1);
            uint32_t it = 0;
            bool ok = true;
            int local = 0;
            const int kt_panel = min(S, KT - 1);
            for (int tile = unit; tile < num_tiles && ok; tile += nunits, ++local) {
                const int tm = tile / tiles_n, tn = tile % tiles_n;
                const int m0 = tm * TM + BM * (int)rank, n0 = tn * BN;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    if (has_lr && kt == kt_panel) {
                        if (!mbar_wait_cluster(&bars[B_LR_SMEM_EMPTY], (local & 1) ^ 1, ERR_WAIT_LR, abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (rank == 0) mbar_arrive_expect_tx(&bars[B_LR_FULL], 2u * lr_share);
                        const LrFactor* fs[2] = {&p.f1, &p.f2};
                        const CUtensorMap* pm[2] = {&p.mapP1, &p.mapP2};
                        const CUtensorMap* lm[2] = {&p.mapL1, &p.mapL2};
                        const uint32_t po[2] = {L.p1, L.p2}, lo[2] = {L.l1, L.l2};
                        for (int f = 0; f < 2; ++f) {
                            const LrFactor& F = *fs[f];
                            for (int a = 0; a < (F.rf > 0 ? F.natoms : 0); ++a) {
                                tma_load_2d_pair(smem + po[f] + a * 128 * F.row_bytes, pm[f], lead_lr,
                                                 F.pcol + 64 * a, m0);
                                for (int h = 0; h < 2; ++h)
                                    tma_load_2d_pair(smem + lo[f] + (a * 128 + h * 64) * F.row_bytes, lm[f], lead_lr,
                                                     64 * a, n0 + 128 * h + 64 * (int)rank);
                            }
                        }
                    }
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait_cluster(&bars[B_EMPTY + s], ph ^ 1, ERR_WAIT_EMPTY, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int blk_row = IMG_BLOCK_ROWS * (tn * KT + kt);
                    uint64_t* sfb_bar = &bars[B_SFFULL + s];
                    mbar_arrive_expect_tx(sfb_bar, SFB_STAGE_BYTES + SFA_STAGE_BYTES);
                    tma_load_2d(smem + L.b + s * B_SLOT_P + B_HALF_BYTES, &p.mapBs, sfb_bar, 0, blk_row + BN);
                    tma_load_3d(smem + L.sfa + s * SFA_STAGE_BYTES, &p.mapSFA, sfb_bar, 0, 8 * kt, 2 * tm + (int)rank);
                    if (rank == 0) mbar_arrive_expect_tx(&bars[B_FULL + s], 2u * (A_BYTES + B_HALF_BYTES));
                    tma_load_2d_pair(smem + L.b + s * B_SLOT_P, &p.mapB, lead_full + 8u * s, 0,
                                     blk_row + (BN / 2) * (int)rank);
                    tma_load_2d_pair(smem + L.a + s * A_BYTES, &p.mapA, lead_full + 8u * s, kt * BK_BYTES, m0);
                }
            }
            if (!ok) {
                // this CTA's scale copies land on its own barriers; its code
                // and panel copies count on the leader's, so give those time
                // to land before the CTA can exit (both CTAs pass a cluster
                // barrier at the end)
                for (int d = 0; d < S && d < (int)it; ++d) {
                    uint32_t j = it - 1 - d;
                    volatile int no_abort = 0;
                    mbar_wait(&bars[B_SFFULL + (j % S)], (j / S) & 1, ERR_WAIT_DRAIN, &no_abort);
                }
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 200000ull) {
                }
            }
        } else if (!kPair && lane == 0) {
            const uint32_t stage_bytes = A_BYTES;
            const uint32_t lr_total = p_bytes(p.f1) + l_bytes(p.f1) + p_bytes(p.f2) + l_bytes(p.f2);
            uint32_t it = 0;
            bool ok = true;
            int local = 0;
            // the tile's low-rank panels are needed only after its mainloop:
            // they are issued once the ring holds the tile's first stages
            // (by then the previous tile's up-projection, their last
            // reader, has been issued), so neither their latency nor that
            // wait holds back the stages
            const int kt_panel = min(S, KT - 1);
            int panels_issued = 0;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits, ++local) {
                const int tm = tile / tiles_n, tn = tile % tiles_n;
                const int m0 = tm * BM, n0 = tn * BN;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    if (has_lr && kt == kt_panel) {
                        if (!mbar_wait(&bars[B_LR_SMEM_EMPTY], (local & 1) ^ 1, ERR_WAIT_LR, abort_flag)) {
                            ok = false;
                            break;
                        }
                        uint64_t* lb = &bars[B_LR_FULL];
                        mbar_arrive_expect_tx(lb, lr_total);
                        for (int a = 0; a < (p.f1.rf > 0 ? p.f1.natoms : 0); ++a) {
                            tma_load_2d(smem + L.p1 + a * 128 * p.f1.row_bytes, &p.mapP1, lb, p.f1.pcol + 64 * a, m0);
                            tma_load_2d(smem + L.l1 + a * 256 * p.f1.row_bytes, &p.mapL1, lb, 64 * a, n0);
                        }
                        for (int a = 0; a < (p.f2.rf > 0 ? p.f2.natoms : 0); ++a) {
                            tma_load_2d(smem + L.p2 + a * 128 * p.f2.row_bytes, &p.mapP2, lb, p.f2.pcol + 64 * a, m0);
                            tma_load_2d(smem + L.l2 + a * 256 * p.f2.row_bytes, &p.mapL2, lb, 64 * a, n0);
                        }
                        ++panels_issued;
                    }
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait(&bars[B_EMPTY + s], ph ^ 1, ERR_WAIT_EMPTY, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (kBf16) {
                        // A [128 rows x 64 columns] and B [256 x 64], bf16
                        uint64_t* fb = &bars[B_FULL + s];
                        mbar_arrive_expect_tx(fb, A_BYTES + B_BYTES);
                        tma_load_2d(smem + L.b + s * B_SLOT, &p.mapB, fb, kt * 64, n0);
                        tma_load_2d(smem + L.a + s * A_BYTES, &p.mapA, fb, kt * 64, m0);
                        continue;
                    }
                    // the weight block (codes and scales in one copy) and the
                    // activation scale slabs first, on their own barrier: the
                    // scale warps stage the scales in tensor memory while the
                    // activation codes are still on their way
                    uint64_t* sfb_bar = &bars[B_SFFULL + s];
                    mbar_arrive_expect_tx(sfb_bar, B_SLOT + SFA_STAGE_BYTES);
                    tma_load_3d(smem + L.b + s * B_SLOT, &p.mapB, sfb_bar, 0, 0, 2 * (tn * KT + kt));
                    tma_load_3d(smem + L.sfa + s * SFA_STAGE_BYTES, &p.mapSFA, sfb_bar, 0, 8 * kt, tm);
                    uint64_t* fb = &bars[B_FULL + s];
                    mbar_arrive_expect_tx(fb, stage_bytes);
                    tma_load_2d(smem + L.a + s * A_BYTES, &p.mapA, fb, kt * BK_BYTES, m0);
                }
            }
            if (!ok && panels_issued > 0) {
                // the last panel copies land before the CTA exits
                volatile int no_abort = 0;
                mbar_wait(&bars[B_LR_FULL], (panels_issued - 1) & 1, ERR_WAIT_DRAIN, &no_abort);
            }
            if (!ok) {
                // let copies already issued land before the CTA exits
                for (int d = 0; d < S && d < (int)it; ++d) {
                    uint32_t j = it - 1 - d;
                    volatile int no_abort = 0;
                    if (!kBf16) mbar_wait(&bars[B_SFFULL + (j % S)], (j / S) & 1, ERR_WAIT_DRAIN, &no_abort);
                    mbar_wait(&bars[B_FULL + (j % S)], (j / S) & 1, ERR_WAIT_DRAIN, &no_abort);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer
        if (kPair && lane == 0 && rank == 0) {
            // the pair's leader: M = 256 MMAs over both CTAs' operands into
            // both CTAs' tensor memory; every completion is committed to
            // the barrier of each CTA that waits for it
            const uint32_t idesc = idesc_nvfp4(2 * BM, BN);
            const uint32_t idesc_lr = idesc_bf16(2 * BM, 128, 0, 0);
            const uint32_t hi_sw128 = (1024u >> 4) | (1u << 14) | (SWZ_128B << 29);
            const uint32_t a_lo0 = ((base + L.a) >> 4) | (1u << 16);
            const uint32_t b_lo0 = ((base + L.b) >> 4) | (1u << 16);
            const uint32_t own0 = smem_u32(&bars[0]);
            const uint32_t peer0 = mapa_shared(own0, 1);
            auto commit_both = [&](int b) {
                tc_commit_pair(own0 + 8u * (uint32_t)b);
                tc_commit_pair(peer0 + 8u * (uint32_t)b);
            };
            uint32_t it = 0;
            // ring positions of `it`, advanced by increments (the MMA
            // thread's per-stage work costs tensor-pipe time; no divisions)
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int local = 0;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits, ++local) {
                // both CTAs' epilogues have read the previous tile
                if (!mbar_wait_cluster(&bars[B_ACC_EMPTY], (local & 1) ^ 1, ERR_WAIT_ACC_EMPTY, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    if (!mbar_wait_cluster(&bars[B_FULL + s], ph, ERR_WAIT_FULL, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_lo = a_lo0 + s * (A_BYTES >> 4);
                    const uint32_t b_lo = b_lo0 + s * (B_SLOT_P >> 4);
                    const uint32_t sf = tmem + RING_COL_P + s * SF_SLOT_COLS;
#pragma unroll
                    for (int j = 0; j < KSTEPS; ++j)
                        umma_nvfp4_pair(tmem + ACC_COL, make_desc(a_lo + 2 * j, hi_sw128),
                                        make_desc(b_lo + 2 * j, hi_sw128), idesc, sf + 4 * j, sf + 16 + 8 * j,
                                        (kt | j) != 0);
                    // the stage's buffers and its scale columns are free again
                    commit_both(B_EMPTY + s);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                commit_both(B_ACC_FULL);
                if (has_lr) {
                    // both halves go into the ring's columns, once the
                    // mainloop's MMAs (their last readers) are done
                    if (!mbar_wait_cluster(&bars[B_LR_FULL], local & 1, ERR_WAIT_LR, abort_flag) ||
                        !mbar_wait_cluster(&bars[B_ACC_FULL], local & 1, ERR_WAIT_ACC_FULL, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    int q = 0;
                    if (p.f1.rf > 0) lr_mma<true>(tmem + LR0_COL, base + L.p1, base + L.l1, p.f1, 0, idesc_lr, q);
                    if (p.f2.rf > 0) lr_mma<true>(tmem + LR0_COL, base + L.p2, base + L.l2, p.f2, 0, idesc_lr, q);
                    commit_both(B_LR0_READY);
                    q = 0;
                    if (p.f1.rf > 0) lr_mma<true>(tmem + R2_COL, base + L.p1, base + L.l1, p.f1, 1, idesc_lr, q);
                    if (p.f2.rf > 0) lr_mma<true>(tmem + R2_COL, base + L.p2, base + L.l2, p.f2, 1, idesc_lr, q);
                    commit_both(B_LR1_READY);
                    commit_both(B_LR_SMEM_EMPTY);
                }
            }
            // every tcgen05 op issued by this thread completes before TMEM is
            // freed and before either CTA can exit
            tc_commit_pair(own0 + 8u * B_DRAIN);
            volatile int no_abort = 0;
            mbar_wait(&bars[B_DRAIN], 0, ERR_WAIT_DRAIN, &no_abort);
        } else if (!kPair && lane == 0) {
            const uint32_t idesc = kBf16 ? idesc_bf16(BM, BN, 0, 0) : idesc_nvfp4(BM, BN);
            const uint32_t idesc_lr = idesc_bf16(BM, 128, 0, 0);
            // descriptor words: lo = start >> 4 | (LBO >> 4) << 16;
            // hi = SBO >> 4 | version 1 << 14 | layout << 29
            const uint32_t hi_sw128 = (1024u >> 4) | (1u << 14) | (SWZ_128B << 29);
            const uint32_t a_lo0 = ((base + L.a) >> 4) | (1u << 16);
            const uint32_t b_lo0 = ((base + L.b) >> 4) | (1u << 16);
            uint32_t it = 0;
            int s = 0;  // it % S and (it / S) & 1, advanced by increments
            uint32_t ph = 0;
            bool ok = true;
            int local = 0;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits, ++local) {
                // the epilogue has read the previous tile's accumulator and
                // both low-rank halves
                if (!mbar_wait(&bars[B_ACC_EMPTY], (local & 1) ^ 1, ERR_WAIT_ACC_EMPTY, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int sb = it & 1;
                    if (!mbar_wait(&bars[B_FULL + s], ph, ERR_WAIT_FULL, abort_flag) ||
                        (!kBf16 && (!mbar_wait(&bars[B_SFFULL + s], ph, ERR_WAIT_FULL, abort_flag) ||
                                    !mbar_wait(&bars[B_SF_READY + sb], (it >> 1) & 1, ERR_WAIT_SF, abort_flag)))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_lo = a_lo0 + s * (A_BYTES >> 4);
                    const uint32_t b_lo = b_lo0 + s * (B_SLOT >> 4);
                    if (kBf16) {
                        // a K = 16 step is 32 bytes of each 128-byte row
#pragma unroll
                        for (int j = 0; j < KSTEPS; ++j)
                            umma_bf16(tmem + ACC_COL, make_desc(a_lo + 2 * j, hi_sw128),
                                      make_desc(b_lo + 2 * j, hi_sw128), idesc, (kt | j) != 0);
                        tc_commit(&bars[B_EMPTY + s]);
                        if (++s == S) {
                            s = 0;
                            ph ^= 1u;
                        }
                        continue;
                    }
                    const uint32_t sf = tmem + R2_COL + sb * SF_SLOT_COLS;
#pragma unroll
                    for (int j = 0; j < KSTEPS; ++j)
                        umma_nvfp4(tmem + ACC_COL, make_desc(a_lo + 2 * j, hi_sw128),
                                   make_desc(b_lo + 2 * j, hi_sw128), idesc, sf + 4 * j, sf + 16 + 8 * j,
                                   (kt | j) != 0);
                    tc_commit(&bars[B_EMPTY + s]);
                    tc_commit(&bars[B_SF_FREE + sb]);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                if (has_lr) {
                    // the up-projection after the mainloop: half 0 at once
                    // (its own columns), half 1 into the scale ring's columns
                    // once the mainloop's MMAs, their last readers, are done
                    if (!mbar_wait(&bars[B_LR_FULL], local & 1, ERR_WAIT_LR, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    int q = 0;
                    if (p.f1.rf > 0) lr_mma<false>(tmem + LR0_COL, base + L.p1, base + L.l1, p.f1, 0, idesc_lr, q);
                    if (p.f2.rf > 0) lr_mma<false>(tmem + LR0_COL, base + L.p2, base + L.l2, p.f2, 0, idesc_lr, q);
                    tc_commit(&bars[B_LR0_READY]);
                }
                tc_commit(&bars[B_ACC_FULL]);
                if (has_lr) {
                    if (!mbar_wait(&bars[B_ACC_FULL], local & 1, ERR_WAIT_ACC_FULL, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    int q = 0;
                    if (p.f1.rf > 0) lr_mma<false>(tmem + R2_COL, base + L.p1, base + L.l1, p.f1, 1, idesc_lr, q);
                    if (p.f2.rf > 0) lr_mma<false>(tmem + R2_COL, base + L.p2, base + L.l2, p.f2, 1, idesc_lr, q);
                    tc_commit(&bars[B_LR1_READY]);
                    tc_commit(&bars[B_LR_SMEM_EMPTY]);
                }
            }
            // every tcgen05 op issued by this thread completes before TMEM is freed
            tc_commit(&bars[B_DRAIN]);
            volatile int no_abort = 0;
            mbar_wait(&bars[B_DRAIN], 0, ERR_WAIT_DRAIN, &no_abort);
        }
        __syncwarp();
    } else if (warp < EPI_WARP0) {
        if constexpr (!kBf16) {  // no block scales in the 16-bit variant
            // ------------------------------------------------ scale warps
            // Warp q (= warp % 4) writes TMEM lanes 32q .. 32q + 31; its lane i
            // stores slab row i of every K step (16 bytes each) into its own
            // lane: the contents a tcgen05.cp 32x128b.warpx4 of each slab would
            // leave in every lane quarter, written by the TMEM store path
            // instead of the tensor pipe.
            const uint32_t lane_addr = (uint32_t)(32 * (warp & 3)) << 16;
            uint32_t it = 0;
            bool ok = true;
            int local = 0;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits, ++local) {
                // the ring's columns hold the previous tile's low-rank half 1
                // until its epilogue (this CTA's) is done
                if (has_lr && local > 0 &&
                    !mbar_wait(&bars[kPair ? B_EPI_DONE : B_ACC_EMPTY], (local - 1) & 1, ERR_WAIT_SF, abort_flag)) {
                    ok = false;
                    break;
                }
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % S;
                    // one-CTA tiles: a two-slot ring freed by the MMAs'
                    // commits; CTA pairs: the stage's own slot, whose last
                    // readers (the MMAs of stage it - S) finished before this
                    // CTA's producer refilled the stage
                    const int sb = kPair ? s : (int)(it & 1);
                    if (!mbar_wait(&bars[B_SFFULL + s], (it / S) & 1, ERR_WAIT_FULL, abort_flag) ||
                        (!kPair && !mbar_wait(&bars[B_SF_FREE + sb], ((it >> 1) & 1) ^ 1, ERR_WAIT_SF, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfa = base + L.sfa + (uint32_t)s * SFA_STAGE_BYTES + 16u * (uint32_t)lane;
                    const uint32_t sfb = kPair ? base + L.b + (uint32_t)s * B_SLOT_P + B_HALF_BYTES + 16u * (uint32_t)lane
                                               : base + L.b + (uint32_t)s * B_SLOT + B_BYTES + 16u * (uint32_t)lane;
                    uint32_t ra[16], rb[32];
    #pragma unroll
                    for (int j = 0; j < KSTEPS; ++j) {
                        const uint4 va = ld_shared_v4(sfa + 512u * j);
                        const uint4 vl = ld_shared_v4(sfb + 512u * j);
                        const uint4 vh = ld_shared_v4(sfb + (uint32_t)SFA_STAGE_BYTES + 512u * j);
                        ra[4 * j] = va.x; ra[4 * j + 1] = va.y; ra[4 * j + 2] = va.z; ra[4 * j + 3] = va.w;
                        rb[8 * j] = vl.x; rb[8 * j + 1] = vl.y; rb[8 * j + 2] = vl.z; rb[8 * j + 3] = vl.w;
                        rb[8 * j + 4] = vh.x; rb[8 * j + 5] = vh.y; rb[8 * j + 6] = vh.z; rb[8 * j + 7] = vh.w;
                    }
                    const uint32_t sf = tmem + lane_addr + (kPair ? RING_COL_P : R2_COL) + (uint32_t)sb * SF_SLOT_COLS;
                    tmem_st_32x32b_x16(sf, ra);
                    tmem_st_32x32b_x32(sf + 16, rb);
                    tmem_st_wait();
                    // the slab bytes were read through the generic proxy; the
                    // stage goes back to TMA after the MMAs
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (kPair) mbar_arrive_cluster(mapa_shared(smem_u32(&bars[B_FULL + sb]), 0));
                        else mbar_arrive(&bars[B_SF_READY + sb]);
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        // Each thread owns one tile row (its TMEM lane) within one of two
        // column groups working concurrently: warps 6-9 take columns 0-127
        // (with low-rank half 0), warps 10-13 columns 128-255 (half 1).
        // Output leaves in chunks of 32 bytes per row (16 bf16 or 8 f32
        // columns): the group's rows are written into its staging buffer
        // (the two 16-byte halves of a row swapped on every other group of
        // four rows, so eight consecutive rows' stores hit distinct banks),
        // then the group copies the 128-row chunk out with 16-byte stores,
        // two threads per row, so every warp store covers whole sectors of
        // sixteen rows.  (A TMA store per chunk would queue in the same copy
        // engine as the next tile's operand loads.)  The small staging
        // buffer keeps three operand stages resident at rank 64.
        const int sp = warp & 3;  // TMEM sub-partition = rows 32*sp .. +31
        const int grp = (warp - EPI_WARP0) >> 2;
        const int et = 32 * sp + lane;  // tile row
        const uint32_t rsw = (uint32_t)((et >> 2) & 1);
        const uint32_t buf = base + L.stg + (uint32_t)grp * STG_BYTES;
        const uint32_t lr_col = grp == 0 ? LR0_COL : R2_COL;
        uint64_t* lr_ready = &bars[grp == 0 ? B_LR0_READY : B_LR1_READY];
        // this warp is done reading the tile's tensor memory: the MMA warp
        // (the pair's leader) may overwrite it, this CTA's scale warps may
        // reuse the ring columns
        auto release_acc = [&]() {
            if (kPair) {
                mbar_arrive(&bars[B_EPI_DONE]);
                mbar_arrive_cluster(mapa_shared(smem_u32(&bars[B_ACC_EMPTY]), 0));
            } else {
                mbar_arrive(&bars[B_ACC_EMPTY]);
            }
        };
        bool ok = true;
        int local = 0;
        const int64_t ldo = (int64_t)p.Nout * (p.out_f32 ? 4 : 2);  // output row bytes
        // running max of |output| over this thread's values (bf16 pairs as
        // two 16-bit lanes, or FP32 bits), for p.amax_out
        uint32_t am2 = 0, am32 = 0;
        // the FP32 tensor scales of the operands (a bf16 activation has none)
        const float gab = p.ga ? __fmul_rn(*p.ga, *p.gb) : *p.gb;
        // MLP fusion: the encode table of Q(H) for the caller's tensor amax,
        // built by the 256 epilogue threads before the first accumulator
        QTableM& tab = *reinterpret_cast<QTableM*>(smem + L.tab);
        uint16_t* gtab = reinterpret_cast<uint16_t*>(smem + L.tab + sizeof(QTableM));
        QTensorFast qt;
        qt.g = qt.six_g = qt.y6 = 0.0f;
        if (kMlp) {
            const int et2 = threadIdx.x - 32 * EPI_WARP0;
            qt = make_qtensor_fast(*p.amax_h);
            build_qtable_m1(tab, qt.g, et2, 32 * NUM_EPI_WARPS);
            named_bar_sync(3, 32 * NUM_EPI_WARPS);
            build_qtable_m2(tab, et2, 32 * NUM_EPI_WARPS);
            named_bar_sync(3, 32 * NUM_EPI_WARPS);
            build_qtable_m3(tab, et2, 32 * NUM_EPI_WARPS);
            named_bar_sync(3, 32 * NUM_EPI_WARPS);
            if (blockIdx.x == 0 && et2 == 0) *p.q_tscale = qt.g;
            // GELU's table (the first tile's mainloop runs meanwhile)
            gelu_table_build(gtab, et2, 32 * NUM_EPI_WARPS);
            named_bar_sync(3, 32 * NUM_EPI_WARPS);
        }
        for (int tile = unit; tile < num_tiles && ok; tile += nunits, ++local) {
            const int m0 = (tile / tiles_n) * TM + BM * (int)rank;
            const int n0 = (tile % tiles_n) * BN;
            if (kPair ? (!mbar_wait_cluster(&bars[B_ACC_FULL], local & 1, ERR_WAIT_ACC_FULL, abort_flag) ||
                         (has_lr && !mbar_wait_cluster(lr_ready, local & 1, ERR_WAIT_LR, abort_flag)))
                      : (!mbar_wait(&bars[B_ACC_FULL], local & 1, ERR_WAIT_ACC_FULL, abort_flag) ||
                         (has_lr && !mbar_wait(lr_ready, local & 1, ERR_WAIT_LR, abort_flag)))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t lane_addr = (uint32_t)(32 * sp) << 16;
            const uint32_t rowa = buf + (uint32_t)et * 32u;
            // stage one 32-byte piece of this thread's row ...
            auto stage = [&](uint4 lo, uint4 hi) {
                st_shared_v4(rowa + (rsw << 4), lo);
                st_shared_v4(rowa + ((rsw ^ 1u) << 4), hi);
            };
            // ... and copy the group's staged chunk at tile column `col` out:
            // piece i is row i / 2, 16-byte half i % 2
            auto copy_out = [&](int col) {
                uint8_t* obase = p.out + (int64_t)m0 * ldo + (int64_t)(n0 + col) * (p.out_f32 ? 4 : 2);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int i = et + 128 * k;
                    const int row = i >> 1, q = i & 1;
                    const uint4 v = ld_shared_v4(buf + (uint32_t)row * 32u +
                                                 (((uint32_t)q ^ (uint32_t)((row >> 2) & 1)) << 4));
                    if (m0 + row < p.M) *reinterpret_cast<uint4*>(obase + (int64_t)row * ldo + 16 * q) = v;
                }
            };
            if (kMlp || !p.out_f32) {
                // bf16: the group's 128 columns of this row are read out of
                // tensor memory and packed first, so the accumulator is
                // released before the stores and the next tile's MMAs run
                // while they drain
                uint32_t pk[8][8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t v[16], lr[16];
                    tmem_ld_32x32b_x16(tmem + lane_addr + ACC_COL + 128 * grp + 16 * c, v);
                    if (has_lr) tmem_ld_32x32b_x16(tmem + lane_addr + lr_col + 16 * c, lr);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float y0 = __fmaf_rn(gab, __uint_as_float(v[2 * k]), has_lr ? __uint_as_float(lr[2 * k]) : 0.0f);
                        const float y1 =
                            __fmaf_rn(gab, __uint_as_float(v[2 * k + 1]), has_lr ? __uint_as_float(lr[2 * k + 1]) : 0.0f);
                        __nv_bfloat162 t = __floats2bfloat162_rn(y0, y1);
                        pk[c][k] = *reinterpret_cast<uint32_t*>(&t);
                        if (!kMlp) am2 = __vmaxu2(am2, pk[c][k] & 0x7FFF7FFFu);
                    }
                }
                // every TMEM read of this tile is done: the MMA warp may
                // overwrite the accumulator and both low-rank halves
                tc_fence_before();
                __syncwarp();
                if (lane == 0) release_acc();
                if (kMlp) {
                    // MLP fusion: H = GELU(y) per bf16 value.  A 16-column
                    // chunk of the row is one 1x16 block of Q(H), and its 32
                    // bytes of H are one whole sector, stored straight from
                    // registers (no staging, no barriers between the group's
                    // warps).
                    const int row = m0 + et;
                    const bool in = row < p.M;
                    const int64_t qcol = n0 + 128 * grp;  // first column of the group
                    uint8_t* hrow = p.out + (int64_t)row * ldo + qcol * 2;
                    uint8_t* crow = p.q_codes + (int64_t)row * (p.Nout / 2) + qcol / 2;
                    uint32_t sw0 = 0, sw1 = 0;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t w[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            w[k] = gelu_bf16x2_tab(pk[c][k], gtab);
                            am2 = __vmaxu2(am2, w[k] & 0x7FFF7FFFu);
                        }
                        uint32_t sbyte;
                        const uint2 q = quant_block16_m(w, amax_bits_16(w), qt, tab, sbyte);
                        if (in) {
                            st_global_v8(hrow + 32 * c, w);
                            *reinterpret_cast<uint2*>(crow + 8 * c) = q;
                        }
                        if (c < 4) sw0 |= sbyte << (8 * c);
                        else sw1 |= sbyte << (8 * (c - 4));
                    }
                    if (in)
                        *reinterpret_cast<uint2*>(p.q_scales + (int64_t)row * (p.Nout / 16) + qcol / 16) =
                            make_uint2(sw0, sw1);
                    // slab rows past M hold the (zero) scales of the zero-filled
                    // rows, up to the slabs' 128-row padding (a pair's second
                    // CTA may lie wholly past it)
                    if (row < ((p.M + BM - 1) / BM) * BM) {
                        *reinterpret_cast<uint32_t*>(p.q_slab + slab_offset(row, qcol / 16, p.Nout)) = sw0;
                        *reinterpret_cast<uint32_t*>(p.q_slab + slab_offset(row, qcol / 16 + 4, p.Nout)) = sw1;
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        // the group's previous chunk has been copied out of the buffer
                        named_bar_sync(1 + grp, 128);
                        stage(make_uint4(pk[c][0], pk[c][1], pk[c][2], pk[c][3]),
                              make_uint4(pk[c][4], pk[c][5], pk[c][6], pk[c][7]));
                        named_bar_sync(1 + grp, 128);
                        copy_out(128 * grp + 16 * c);
                    }
                }
            } else {
                // FP32: eight reads of 16 columns, each leaving as two chunks
                // of 8; the accumulator released after the last
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    const int lcol = 16 * c;          // column within the group's half
                    const int col = 128 * grp + lcol; // tile column
                    uint32_t v[16], lr[16];
                    tmem_ld_32x32b_x16(tmem + lane_addr + ACC_COL + col, v);
                    if (has_lr) tmem_ld_32x32b_x16(tmem + lane_addr + lr_col + lcol, lr);
                    tmem_ld_wait();
                    uint32_t y[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                    {
                        y[k] = __float_as_uint(
                            __fmaf_rn(gab, __uint_as_float(v[k]), has_lr ? __uint_as_float(lr[k]) : 0.0f));
                        am32 = max(am32, y[k] & 0x7FFFFFFFu);
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        named_bar_sync(1 + grp, 128);
                        stage(make_uint4(y[8 * h], y[8 * h + 1], y[8 * h + 2], y[8 * h + 3]),
                              make_uint4(y[8 * h + 4], y[8 * h + 5], y[8 * h + 6], y[8 * h + 7]));
                        named_bar_sync(1 + grp, 128);
                        copy_out(col + 8 * h);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) release_acc();
            }
        }
        if (p.amax_out) {
            // rows past M and padding columns hold zeros; one reduction per
            // warp and launch (non-negative floats order like their bits)
            uint32_t a = max(max(am2 & 0xFFFFu, am2 >> 16) << 16, am32);
            a = __reduce_max_sync(0xFFFFFFFFu, a);
            if (lane == 0 && a != 0u) atomicMax(p.amax_out, a);
        }
    }

    tc_fence_before();
    __syncthreads();
    // neither CTA of a pair leaves while the other may still read its shared
    // memory or signal its barriers
    if constexpr (kPair) cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        if (kPair) tmem_dealloc_pair(tmem, TMEM_COLS);
        else tmem_dealloc(tmem, TMEM_COLS);
    }
    finish_after_predecessor(p.dep_done);
}

}  // namespace gemm
}  // namespace ft
