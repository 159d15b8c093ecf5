// k_lora_grad.cuh -- adapter weight gradients (FourTune page, section 3.2:
// weight gradients only for the trainable branch, dB = (X A)^T G and
// dA = X^T (G B^T) in the page's notation).  With the saved, already scaled
// P_lora = bf16(s X A) and Pg_lora = bf16(s dY B):
//     dB[n, j] = sum_m dY[m, n] P_lora[m, j]        (z = 0)
//     dA[k, j] = sum_m X[m, k]  Pg_lora[m, j]       (z = 1)
// Both are out[c, j] = sum_m T[m, c] S[m, j]: a reduction over the token
// dimension, HBM-bound on reading T.  Each CTA takes 128 columns c and a
// slice of m, runs tcgen05 kind::f16 with both operands MN-major straight
// from the TMA tiles (T^T as A, S as B), and writes an FP32 partial; the last
// CTA of a column tile (completion counter) adds the slices in split order
// into the output.  A stage is 128 token rows: T arrives as one 32 KB 3-D
// box (both 64-column halves) and S as one 16 KB box per 64 columns, since
// the copy engine's cost is per copy far more than per byte.
#pragma once

#include <cuda.h>

#include "ft_ptx.cuh"

namespace ft {
namespace lgrad {

constexpr int BC = 128;    // output rows (columns of T) per CTA
constexpr int BMR = 128;   // token rows per stage
constexpr int MAX_STAGES = 4;
constexpr int MAX_SPLITS = 16;  // token slices of one column tile
constexpr int NUM_THREADS = 192;
constexpr int T_BYTES = BMR * BC * 2;    // 32 KiB: two 64-column swizzle atoms
constexpr int S_CHUNK = BMR * 64 * 2;    // 16 KiB: one 64-column box
constexpr uint32_t TMEM_COLS = 128;

struct Params {
    CUtensorMap mapT[2];  // bf16 [M, C_z] as {64, M, C_z / 64}, box {64, 128, 2}, 128 B swizzle
    CUtensorMap mapS[2];  // bf16 [M, r],   box {64, 128}, 128 B swizzle
    float* part[2];       // [splits, C_z, r_l]
    float* out[2];        // dB [N, r_l], dA [K, r_l]
    unsigned long long* counters;  // [2][ctiles_max] epoch-tagged arrivals of the splits
    unsigned long long epoch;      // this launch's epoch (host-issued, increasing)
    const unsigned long long* dep_done;  // null, or the finished-CTA counter of the kernel that wrote S,
    unsigned long long dep_epoch;        // its epoch
    unsigned int dep_count;              // and its grid size
    int C[2];
    int M, r_s, r_l, n_pad, mrows, splits, ctiles_max;
    int stages;
};

// Stages that fit 192 KiB of ring: four with one S box, three with two.
constexpr int stages_for(int n_pad) {
    return (192 * 1024) / (T_BYTES + (n_pad / 64) * S_CHUNK) > MAX_STAGES
               ? MAX_STAGES
               : (192 * 1024) / (T_BYTES + (n_pad / 64) * S_CHUNK);
}
constexpr uint32_t smem_bytes(int n_pad) {
    return stages_for(n_pad) * (T_BYTES + (n_pad / 64) * S_CHUNK) + 256 + 1024;
}

// out = the sum over splits of the partials, in split order, for n4 float4
// elements; every split's loads of UNR elements are in flight together.
template <int MAXS, int UNR>
__device__ __forceinline__ void reduce_splits(const float4* part4, int64_t stride4, int n4, int splits,
                                              float4* out4) {
    for (int i0 = threadIdx.x; i0 < n4; i0 += UNR * NUM_THREADS) {
        float4 v[UNR][MAXS];
#pragma unroll
        for (int k = 0; k < MAXS; ++k) {
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int i = i0 + u * NUM_THREADS;
                v[u][k] = (k < splits && i < n4) ? __ldcg(part4 + k * stride4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int i = i0 + u * NUM_THREADS;
            if (i >= n4) continue;
            float4 acc = v[u][0];
#pragma unroll
            for (int k = 1; k < MAXS; ++k) {
                if (k < splits) {
                    acc.x = __fadd_rn(acc.x, v[u][k].x);
                    acc.y = __fadd_rn(acc.y, v[u][k].y);
                    acc.z = __fadd_rn(acc.z, v[u][k].z);
                    acc.w = __fadd_rn(acc.w, v[u][k].w);
                }
            }
            out4[i] = acc;
        }
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) k_lora_grad(const __grid_constant__ Params p) {
    const int z = blockIdx.z;
    const int c0 = blockIdx.x * BC;
    if (c0 >= p.C[z]) return;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const int nsc = p.n_pad / 64;
    const uint32_t s_bytes = nsc * S_CHUNK;
    const int STAGES = p.stages;
    const uint32_t off_t = 0, off_s = STAGES * T_BYTES, off_bar = STAGES * (T_BYTES + s_bytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + off_bar);
    uint64_t* empty = full + MAX_STAGES;
    uint64_t* accfull = empty + MAX_STAGES;
    uint64_t* drain = accfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;

    const int warp = warp_id(), lane = lane_id();
    const int split = blockIdx.y;
    const int mbeg = split * p.mrows;
    const int mend = min(p.M, mbeg + p.mrows);
    const int nst = mend > mbeg ? (mend - mbeg + BMR - 1) / BMR : 0;
    const CUtensorMap* mapT = &p.mapT[z];
    const CUtensorMap* mapS = &p.mapS[z];

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(accfull, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the inputs written by the previous kernel are complete from here on;
    // the next kernel may start its own setup
    wait_inputs(p.dep_done, p.dep_epoch, p.dep_count, abort_flag);

    if (warp == 0) {
        if (lane == 0) {
            int st = 0;
            for (; st < nst; ++st) {
                const int s = st % STAGES;
                const uint32_t ph = (st / STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, ERR_WAIT_EMPTY, abort_flag)) break;
                const int m = mbeg + st * BMR;
                mbar_arrive_expect_tx(&full[s], T_BYTES + s_bytes);
                tma_load_3d(smem + off_t + s * T_BYTES, mapT, &full[s], 0, m, c0 / 64);
                uint8_t* sdst = smem + off_s + s * s_bytes;
                for (int h = 0; h < nsc; ++h)
                    tma_load_2d(sdst + h * S_CHUNK, mapS, &full[s], p.r_s + 64 * h, m);
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
        if (lane == 0) {
            // A = T^T (M = 128 columns c, MN-major: two 64-wide swizzle atoms
            // 8 KiB apart), B = S (N = n_pad, MN-major), K = 16 token rows.
            const uint32_t idesc = idesc_bf16(BC, p.n_pad, 1, 1);
            // descriptor words built once (lo = start >> 4 | (LBO >> 4) << 16,
            // hi = SBO >> 4 | version 1 << 14 | swizzle << 29): atoms / boxes
            // LBO apart, 8-row groups 1 KiB apart; a K step is 16 rows (2 KiB)
            const uint32_t hi = (1024u >> 4) | (1u << 14) | (SWZ_128B << 29);
            const uint32_t a_lo0 = ((base + off_t) >> 4) | ((uint32_t)((T_BYTES / 2) >> 4) << 16);
            const uint32_t b_lo0 = ((base + off_s) >> 4) | ((uint32_t)(S_CHUNK >> 4) << 16);
            bool ok = true;
            for (int st = 0; st < nst; ++st) {
                const int s = st % STAGES;
                const uint32_t ph = (st / STAGES) & 1;
                if (!mbar_wait(&full[s], ph, ERR_WAIT_FULL, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_lo = a_lo0 + (uint32_t)s * (T_BYTES >> 4);
                const uint32_t b_lo = b_lo0 + (uint32_t)s * (s_bytes >> 4);
#pragma unroll
                for (int k = 0; k < BMR / 16; ++k)
                    umma_bf16(tmem, make_desc(a_lo + 128 * k, hi), make_desc(b_lo + 128 * k, hi), idesc,
                              (st | k) != 0);
                tc_commit(&empty[s]);
            }
            if (ok && nst > 0) tc_commit(accfull);
            tc_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, ERR_WAIT_DRAIN, &no_abort);
        }
        __syncwarp();
    } else {
        const int sp = warp & 3;
        const int c = c0 + 32 * sp + lane;
        float* out = p.part[z] + ((int64_t)split * p.C[z] + c) * p.r_l;
        bool have = nst > 0 && mbar_wait(accfull, 0, ERR_WAIT_ACC_FULL, abort_flag);
        if (have) tc_fence_after();
        const uint32_t lane_addr = (uint32_t)(32 * sp) << 16;
        for (int j0 = 0; j0 < p.r_l; j0 += 32) {
            uint32_t v[32];
            if (have) {
                tmem_ld_32x32b_x32(tmem + lane_addr + j0, v);
                tmem_ld_wait();
            }
#pragma unroll
            for (int k = 0; k < 32; ++k)
                if (j0 + k < p.r_l) out[j0 + k] = have ? __uint_as_float(v[k]) : 0.0f;
        }
    }
    // every thread's partial writes become visible device-wide before the
    // completion counter below is bumped
    __threadfence();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    bool last = false;
    if (!*abort_flag) {
        if (threadIdx.x == 0) {
            __threadfence();
            const unsigned long long prev = epoch_count(&p.counters[z * p.ctiles_max + blockIdx.x], p.epoch);
            *last_flag = (prev == (unsigned long long)(p.splits - 1)) ? 1 : 0;
        }
        __syncthreads();
        last = *last_flag != 0;
    }
    if (last) {
        __threadfence();
        // the tile's partials, 4 floats at a time: every split's load of UNR
        // elements is issued before the first add (one L2 round trip per
        // pass), then the adds run in split order
        const int n4 = BC * p.r_l / 4;
        const int64_t stride4 = (int64_t)p.C[z] * p.r_l / 4;
        const float4* part4 = reinterpret_cast<const float4*>(p.part[z]) + (int64_t)c0 * p.r_l / 4;
        float4* out4 = reinterpret_cast<float4*>(p.out[z]) + (int64_t)c0 * p.r_l / 4;
        if (p.splits <= 4)
            reduce_splits<4, 3>(part4, stride4, n4, p.splits, out4);
        else
            reduce_splits<MAX_SPLITS, 1>(part4, stride4, n4, p.splits, out4);
    }
    // this grid completes only after the dgrad GEMM it overlapped
    finish_after_predecessor(p.dep_done);
}

}  // namespace lgrad

}  // namespace ft
