// ft_api.cu -- the C ABI declared in include/ft.h.  Host-side argument
// validation, workspace planning, TMA descriptor encoding and kernel
// launches.  The kernels live in the included .cuh files (one translation
// unit, so the device error word is a single symbol).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/ft.h"
#include "ft_nvfp4.cuh"
#include "ft_ptx.cuh"
#include "k_gemm_fp4.cuh"
#include "k_lora_grad.cuh"
#include "k_qdown.cuh"
#include "k_qres.cuh"
#include "k_quant.cuh"

namespace {

using ft::gemm::Params;

// ------------------------------------------------------------ device info
struct DevInfo {
    bool init = false;
    bool ok = false;
    int sms = 0;
    bool attr_set = false;
    int qres_ctas = 0;  // CTAs of k_qres that fit on the device at once
    unsigned long long ctx = 0;  // the context the kernel attributes were set in
};
DevInfo g_dev[64];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;

// The unique ID of the current device's context (the primary context the
// runtime uses).  Per-device state the library caches -- kernel attributes,
// the device address of a module variable -- belongs to one context;
// cudaDeviceReset destroys it, and the next context has a new ID.  Caller
// holds g_mu.
ft_status current_ctx_id(int dev, unsigned long long* id) {
    if (!g_ctx_current || !g_ctx_id) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || !f1 ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess || !f2)
            return FT_ERR_CUDA;
        g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
        g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
    }
    CUcontext c = nullptr;
    if (g_ctx_current(&c) != CUDA_SUCCESS) return FT_ERR_CUDA;
    if (!c) {
        // no context current yet: cudaSetDevice initialises the runtime's
        // primary context of the device and makes it current
        if (cudaSetDevice(dev) != cudaSuccess || g_ctx_current(&c) != CUDA_SUCCESS || !c) return FT_ERR_CUDA;
    }
    return g_ctx_id(c, id) == CUDA_SUCCESS ? FT_OK : FT_ERR_CUDA;
}

ft_status device_info(DevInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo& d = g_dev[dev];
    unsigned long long ctx = 0;
    if (current_ctx_id(dev, &ctx) != FT_OK) return FT_ERR_CUDA;
    if (d.attr_set && d.ctx != ctx) d.attr_set = false;  // a new context: set the attributes again
    if (!d.init) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FT_ERR_CUDA;
        d.ok = (major == 10 && minor == 0);
        d.sms = sms;
        d.init = true;
    }
    if (!d.ok) return FT_ERR_UNSUPPORTED;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return FT_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (!d.attr_set) {
        const int big = 227 * 1024;
        if (cudaFuncSetAttribute(ft::gemm::k_gemm_fp4<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 big) != cudaSuccess ||
            cudaFuncSetAttribute(ft::gemm::k_gemm_fp4<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 big) != cudaSuccess ||
            cudaFuncSetAttribute(ft::gemm::k_gemm_fp4<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 big) != cudaSuccess ||
            cudaFuncSetAttribute(ft::gemm::k_gemm_fp4<false, false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, big) != cudaSuccess ||
            cudaFuncSetAttribute(ft::gemm::k_gemm_fp4<false, true, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, big) != cudaSuccess ||
            cudaFuncSetAttribute(ft::qdown::k_qdown, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ft::qdown::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(ft::lgrad::k_lora_grad, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ft::lgrad::smem_bytes(128)) != cudaSuccess ||
            cudaFuncSetAttribute(ft::qres::k_qres, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 big) != cudaSuccess)
            return FT_ERR_CUDA;
        // one shared-memory carveout (the largest) for every kernel of a
        // step, so that no SM has to re-partition L1 between two of them
        const void* kernels[] = {
            reinterpret_cast<const void*>(ft::gemm::k_gemm_fp4<false>),
            reinterpret_cast<const void*>(ft::gemm::k_gemm_fp4<true>),
            reinterpret_cast<const void*>(ft::gemm::k_gemm_fp4<false, true>),
            reinterpret_cast<const void*>(ft::gemm::k_gemm_fp4<false, false, true>),
            reinterpret_cast<const void*>(ft::gemm::k_gemm_fp4<false, true, true>),
            reinterpret_cast<const void*>(ft::qres::k_qres),
            reinterpret_cast<const void*>(ft::qdown::k_qdown),
            reinterpret_cast<const void*>(ft::lgrad::k_lora_grad),
            reinterpret_cast<const void*>(ft::k_amax_bf16),
            reinterpret_cast<const void*>(ft::k_quant_1x16),
            reinterpret_cast<const void*>(ft::k_pack_lt),
        };
        for (const void* k : kernels)
            if (cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
                return FT_ERR_CUDA;
        // the resident quantizer's grid barrier needs every CTA resident at
        // once; size its grids by the occupancy at its largest footprint
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &per_sm, ft::qres::k_qres, ft::qres::NUM_THREADS, ft::qres::SMEM_LIMIT) != cudaSuccess)
            return FT_ERR_CUDA;
        d.qres_ctas = per_sm * d.sms;
        d.attr_set = true;
        d.ctx = ctx;
    }
    *out = &d;
    return FT_OK;
}

inline ft_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? FT_OK : FT_ERR_CUDA; }
inline ft_status last_launch() { return cuda_ok(cudaGetLastError()); }

// Launches `kernel` so that it may begin while the previous kernel on the
// stream finishes (programmatic stream serialization): the kernel waits for
// that kernel's results itself (grid_dep_wait) after its setup.
// cluster_x > 1: thread-block clusters of that many CTAs along x (the
// GEMM's CTA pairs).
template <typename P>
ft_status launch_overlapped(void (*kernel)(P), dim3 grid, dim3 block, size_t smem, cudaStream_t st, const P& p,
                            int cluster_x = 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 1;
    if (cluster_x > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)cluster_x;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    cfg.attrs = attr;
    return cuda_ok(cudaLaunchKernelEx(&cfg, kernel, p));
}
// The same launch for a kernel taking plain arguments.
template <typename... KArgs, typename... Args>
ft_status launch_overlapped_args(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_ok(cudaLaunchKernelEx(&cfg, kernel, args...));
}
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline int cdiv(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

#define FT_TRY(expr)                 \
    do {                             \
        ft_status _s = (expr);       \
        if (_s != FT_OK) return _s;  \
    } while (0)

// ------------------------------------------------------------ kernel timing
// Optional measurement support: when enabled, every launch is bracketed by a
// pair of CUDA events on its stream; ft_timing_read() adds up the elapsed
// times per kernel.  Disabled by default (zero cost beyond a flag test).
enum KernelId {
    KID_AMAX = 0,
    KID_QUANT_1X16,
    KID_QUANT_TILE16,
    KID_PACK_LT,
    KID_QDOWN,
    KID_LR_FINALIZE,
    KID_GEMM,
    KID_LORA_GRAD,
    KID_LORA_REDUCE,
    KID_QRES,
    KID_GEMM_BF16,
    KID_DEQUANT_W,
    KID_GELU,
    KID_COUNT
};
const char* const kKernelNames[KID_COUNT] = {
    "k_amax_bf16", "k_quant_1x16", "k_quant_tile16", "k_pack_lt", "k_qdown",
    "k_lowrank_finalize", "k_gemm_fp4", "k_lora_grad", "k_lora_grad_reduce", "k_qres",
    "k_gemm_bf16", "k_dequant_w", "k_gelu_bf16"};

struct TimingRec {
    cudaEvent_t a, b;
    int kid;
};
struct Timing {
    bool on = false;
    std::vector<TimingRec> recs;
    std::vector<cudaEvent_t> pool;
    double ms[KID_COUNT] = {};
    int64_t launches[KID_COUNT] = {};
    std::mutex mu;
} g_timing;

cudaEvent_t timing_event() {
    if (!g_timing.pool.empty()) {
        cudaEvent_t e = g_timing.pool.back();
        g_timing.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Brackets one launch: construct before it, call stop() after it.
struct LaunchTimer {
    int kid;
    cudaStream_t st;
    cudaEvent_t a = nullptr;
    LaunchTimer(int k, cudaStream_t s) : kid(k), st(s) {
        if (!g_timing.on) return;
        std::lock_guard<std::mutex> lk(g_timing.mu);
        a = timing_event();
        cudaEventRecord(a, st);
    }
    void stop() {
        if (!a) return;
        std::lock_guard<std::mutex> lk(g_timing.mu);
        cudaEvent_t b = timing_event();
        cudaEventRecord(b, st);
        g_timing.recs.push_back({a, b, kid});
        a = nullptr;
    }
};

// ------------------------------------------------------------ tensor maps
ft_status encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swz) {
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FT_OK : FT_ERR_CUDA;
}

// A row-major bf16 matrix [rows, cols] as the 3-D tensor {64, rows, cols / 64}
// (64-column blocks as the outer dimension), boxes {64, box_rows, depth}:
// `depth` side-by-side 128-byte-swizzled 64-column tiles in one copy.
ft_status encode_colblocks(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_rows,
                           uint32_t depth) {
    cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
    cuuint64_t strides[2] = {(cuuint64_t)(cols * 2), 128};
    cuuint32_t box[3] = {64, box_rows, depth};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FT_OK : FT_ERR_CUDA;
}

// Scale slabs [tiles][k-steps][512 B] as a 3-D byte tensor {256, 2 * k-steps,
// tiles} with boxes of {256, 8, depth}: one stage's four slabs of `depth`
// consecutive 128-row tiles per copy.
ft_status encode_slabs(CUtensorMap* m, const uint8_t* slabs, int64_t ksteps, int64_t tiles, uint32_t depth) {
    cuuint64_t dims[3] = {256, (cuuint64_t)(2 * ksteps), (cuuint64_t)tiles};
    cuuint64_t strides[2] = {256, (cuuint64_t)(ksteps * 512)};
    cuuint32_t box[3] = {256, 8, depth};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(slabs), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FT_OK : FT_ERR_CUDA;
}

// ------------------------------------------------------------ workspace
constexpr int QD_MAX_SPLITS = 8;
constexpr int QRES_MAX_ROW_TILES = 1024;  // row tiles the resident quantizer's counters cover
constexpr int LG_MAX_CTILES = 8192;       // column tiles of the adapter gradients (C <= 2^20)
constexpr int LG_MAX_SPLITS = 16;
static_assert(QD_MAX_SPLITS <= ft::qres::MAX_SPLITS, "k_qres reduces at most MAX_SPLITS partials");
static_assert(LG_MAX_SPLITS <= ft::lgrad::MAX_SPLITS, "k_lora_grad reduces at most MAX_SPLITS partials");

struct WsPlan {
    size_t amax, gact, codes, scales, sfslab, lt, part, pg, lgpart, sync, qcnt, lgcnt, counters, total;
    int n_qd_counters, lg_ctiles;
    // sync: the resident quantizer's epoch-tagged words (grid-barrier
    // arrivals, tensor amax, finished CTAs); qcnt: its row-tile counters;
    // lgcnt: the adapter-gradient tile counters (all epoch-tagged: no reset);
    // counters: the streaming quantizer's row-tile counters (zeroed per call)
};

// A kernel whose every CTA counts itself into the epoch-tagged word `done`
// when its writes are finished; the kernel after it waits for `count` at
// `epoch` instead of the grid's end.
struct DepFlag {
    const unsigned long long* done = nullptr;
    unsigned long long epoch = 0;
    unsigned int count = 0;
};

// Epochs for the epoch-tagged counters: increasing across every launch of
// the process.  The start is taken from the clock (below 2^28) so that a
// word holding a foreign value is unlikely to match; the amax word keeps
// 33 bits of epoch, about 8e9 launches.
unsigned long long next_epoch() {
    static std::atomic<unsigned long long> e{
        (unsigned long long)(std::chrono::steady_clock::now().time_since_epoch().count() >> 10) &
        ((1ull << 28) - 1)};
    return ++e;
}

WsPlan plan_ws(int64_t M, int64_t N, int64_t K, int64_t r_s, int64_t r_l) {
    WsPlan w;
    const int64_t C = std::max(N, K);
    const int64_t r = r_s + r_l;
    size_t o = 0;
    // The epoch-tagged words come first, at offsets no shape changes, so a
    // workspace shared by calls of different shapes only ever holds epoch
    // counters there (their content from any earlier call is valid).
    w.sync = o;   o += 256;
    w.qcnt = o;   o += (size_t)QRES_MAX_ROW_TILES * 8;
    w.lgcnt = o;  o += (size_t)2 * LG_MAX_CTILES * 8;
    w.amax = o;   o += 256;
    w.gact = o;   o += 256;
    w.codes = o;  o += up256((size_t)M * C / 2);
    w.scales = o; o += up256((size_t)M * C / 16);
    w.sfslab = o; o += up256((size_t)((M + 127) / 128) * 128 * C / 16);  // GEMM scale slabs
    w.lt = o;     o += up256((size_t)128 * C * 2);
    w.part = o;   o += up256((size_t)QD_MAX_SPLITS * M * r * 4);
    w.pg = o;     o += up256((size_t)M * r * 2);
    w.lgpart = o; o += up256((size_t)LG_MAX_SPLITS * (N + K) * r_l * 4);
    // completion counters: one per row tile of the fused quantize/down-proj,
    // one per (gradient, column tile) of the adapter gradients
    w.n_qd_counters = (int)((M + 127) / 128);
    w.lg_ctiles = (int)((C + 127) / 128);
    w.counters = o; o += up256((size_t)w.n_qd_counters * 4);
    w.total = o;
    return w;
}

// ------------------------------------------------------------ pieces
ft_status run_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, float* slot, const DevInfo* d,
                   cudaStream_t st) {
    // slot: the first half of an 8-byte-aligned 64-bit word that the kernel
    // tags with this launch's epoch (no clearing, no memset between kernels)
    if (reinterpret_cast<uintptr_t>(slot) & 7u) return FT_ERR_ALIGN;
    const int64_t vecs = rows * (cols / 8);
    // a few CTAs per SM, each thread looping with eight 16-byte loads in
    // flight: every CTA ends in one same-address atomic, which serialise in
    // L2, so thousands of short CTAs would queue on it
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(vecs, 8 * 256), (int64_t)d->sms * 4));
    {
        LaunchTimer _lt(KID_AMAX, st);
        FT_TRY(launch_overlapped_args(ft::k_amax_bf16, dim3((unsigned)grid), dim3(256), 0, st,
                                 static_cast<const uint16_t*>(x), rows, cols, ld,
                                 reinterpret_cast<unsigned long long*>(slot), next_epoch()));
        _lt.stop();
    }
    return last_launch();
}

ft_status run_quant_1x16(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* amax,
                         uint8_t* codes, uint8_t* scales, float* tscale, uint8_t* slab,
                         const DevInfo* d, cudaStream_t st) {
    const int64_t blocks = rows * (cols / 16);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(blocks, 256), (int64_t)d->sms * 16));
    {
        LaunchTimer _lt(KID_QUANT_1X16, st);
        ft::k_quant_1x16<<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), rows, cols, ld, amax,
                                               codes, scales, tscale, slab);
        _lt.stop();
    }
    return last_launch();
}

ft_status run_tile16(bool mode16x16, const void* x, int64_t rows, int64_t cols, int64_t ld,
                     const float* amax, uint8_t* codes_row, uint8_t* scales_row, uint8_t* codes_col,
                     uint8_t* scales_col, float* tscale, float* tscale2, const DevInfo* d, cudaStream_t st) {
    // persistent CTAs over the 64 x 128 tiles, a few per SM
    const int64_t tiles = ((rows + 63) / 64) * ((cols + 127) / 128);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, (int64_t)d->sms * 6));
    LaunchTimer _lt(KID_QUANT_TILE16, st);
    if (mode16x16)
        ft::k_quant_tile16<true><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), rows, cols, ld, amax,
                                                       codes_row, scales_row, codes_col, scales_col, tscale,
                                                       tscale2);
    else
        ft::k_quant_tile16<false><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), rows, cols, ld, amax,
                                                        codes_row, scales_row, codes_col, scales_col, tscale,
                                                        tscale2);
    _lt.stop();
    return last_launch();
}

// Q(T) and P = [bf16(T L1) | bf16(s T L2)] in one pass over T [M, C].
// Also zeroes its row-tile completion counters.
// quant = false: P alone (T's quantized form is produced elsewhere).
ft_status run_qdown(const void* T, int64_t M, int64_t C, const void* L1, int64_t r1, const void* L2,
                    int64_t r2, float s, const float* amax, uint8_t* codes, uint8_t* scales,
                    float* tscale, void* P, uint8_t* ws, const WsPlan& w, const DevInfo* d,
                    cudaStream_t st, bool quant = true) {
    const int64_t r = r1 + r2;
    uint8_t* slab = ws + w.sfslab;
    if (r == 0) return quant ? run_quant_1x16(T, M, C, C, amax, codes, scales, tscale, slab, d, st) : FT_OK;
    float* part = reinterpret_cast<float*>(ws + w.part);
    unsigned int* counters = reinterpret_cast<unsigned int*>(ws + w.counters);
    FT_TRY(cuda_ok(cudaMemsetAsync(counters, 0, (size_t)w.n_qd_counters * 4, st)));
    ft::qdown::Params p;
    std::memset(&p, 0, sizeof(p));
    p.direct = (r1 <= 64 && r2 <= 64) ? 1 : 0;
    if (p.direct) {
        if (r1 > 0)
            FT_TRY(encode_2d(&p.mapL1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1, r1, C, r1 * 2, 64, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B));
        if (r2 > 0)
            FT_TRY(encode_2d(&p.mapL2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2, r2, C, r2 * 2, 64, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B));
    } else {
        uint16_t* Lt = reinterpret_cast<uint16_t*>(ws + w.lt);
        dim3 grid((unsigned)cdiv(C, 256), 128);
        {
            LaunchTimer _lt(KID_PACK_LT, st);
            ft::k_pack_lt<<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(L1), (int)r1,
                                                static_cast<const uint16_t*>(L2), (int)r2, (int)C, Lt);
            _lt.stop();
        }
        FT_TRY(last_launch());
        FT_TRY(encode_2d(&p.mapL1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Lt, C, 128, C * 2, 64, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B));
    }
    const int mt = cdiv(M, ft::qdown::BM);
    int splits = std::max(1, std::min(QD_MAX_SPLITS, d->sms / std::max(1, mt)));
    int cchunk = cdiv(C, (int64_t)splits * 64) * 64;
    splits = cdiv(C, cchunk);
    FT_TRY(encode_2d(&p.mapT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, T, C, M, C * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B));
    p.amax = amax;
    p.tscale = tscale;
    p.codes = codes;
    p.scales = scales;
    p.slab = slab;
    p.part = part;
    p.P = static_cast<__nv_bfloat16*>(P);
    p.counters = counters;
    p.M = (int)M;
    p.C = (int)C;
    p.r = (int)r;
    p.r1 = (int)r1;
    p.cchunk = cchunk;
    p.splits = splits;
    p.s = s;
    p.do_mma = 1;
    p.quant = quant ? 1 : 0;
    {
        LaunchTimer _lt(KID_QDOWN, st);
        ft::qdown::k_qdown<<<dim3((unsigned)mt, (unsigned)splits), ft::qdown::NUM_THREADS,
                             ft::qdown::SMEM_BYTES, st>>>(p);
        _lt.stop();
    }
    return last_launch();
}

// Factor tile of the resident quantizer for a rank rf (a multiple of 16):
// rf / 16 atoms of 16 columns x 64 rows.
ft::qres::Factor qres_factor(int64_t rf) {
    ft::qres::Factor f;
    std::memset(&f, 0, sizeof(f));
    f.rf = (int)std::max<int64_t>(rf, 0);
    return f;
}
uint32_t qres_factor_bytes(const ft::qres::Factor& f) {
    return (uint32_t)(f.rf / 16) * ft::qres::ATOM_BYTES;
}

// L [C, rf] row-major as the 3-D tensor {16, C, rf / 16} (16-column atoms as
// the outer dimension), boxes {16, 64, rf / 16}: a stage's atoms in one copy.
ft_status encode_factor_atoms(CUtensorMap* m, const void* L, int64_t C, int64_t rf) {
    cuuint64_t dims[3] = {16, (cuuint64_t)C, (cuuint64_t)(rf / 16)};
    cuuint64_t strides[2] = {(cuuint64_t)(rf * 2), 32};
    cuuint32_t box[3] = {16, 64, (cuuint32_t)(rf / 16)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(L), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FT_OK : FT_ERR_CUDA;
}

// Ring of factor tiles: as many stages of both tiles as fit in 31 KiB (the
// room left beside 12 resident 16 KiB stages; at least 2 stages), and at
// least the 6 KiB the staged scales need.
void qres_ring(ft::qres::Params& p) {
    namespace Q = ft::qres;
    p.f1.off = 0;
    p.f2.off = qres_factor_bytes(p.f1);
    p.fstage_bytes = qres_factor_bytes(p.f1) + qres_factor_bytes(p.f2);
    // 24 KB of ring leaves room for twelve resident 16 KB stages (a
    // [128, 768] chunk) next to the scale staging, the table and the barriers
    p.fs = 2;
    if (p.fstage_bytes > 0)
        p.fs = (int)std::max<uint32_t>(2u, std::min<uint32_t>((uint32_t)Q::MAX_FS, 24576u / p.fstage_bytes));
    p.ring_bytes = ((uint32_t)p.fs * p.fstage_bytes + 1023u) & ~1023u;
}

// Grid of the resident quantizer for T [M, C]: 128-row tiles x C-splits of
// at most max_st 64-column stages; false when the chunks do not all fit on
// the device at once.
bool qres_grid(int64_t M, int64_t C, int max_st, const DevInfo* d, int* mt, int* splits, int* cchunk) {
    namespace Q = ft::qres;
    if (C % Q::BKC || max_st < 1) return false;
    *mt = cdiv(M, Q::BM);
    int sp = std::max(1, std::min(QD_MAX_SPLITS, d->sms / std::max(1, *mt)));
    sp = std::max(sp, cdiv(C, (int64_t)max_st * Q::BKC));
    *cchunk = cdiv(C, (int64_t)sp * Q::BKC) * Q::BKC;
    *splits = cdiv(C, *cchunk);
    return *splits <= QD_MAX_SPLITS && *cchunk <= max_st * Q::BKC &&
           (int64_t)(*mt) * (*splits) <= d->qres_ctas;
}

// Resident stages that fit next to the ring, the table and the barriers.
int qres_max_stages(uint32_t ring_bytes) {
    namespace Q = ft::qres;
    const int64_t avail = (int64_t)Q::SMEM_LIMIT - Q::make_layout(0, ring_bytes).total;
    return (int)std::min<int64_t>(Q::MAX_ST, std::max<int64_t>(0, avail / Q::TILE_BYTES));
}

// Launch mode of k_qres when it computes the tensor amax (its grid barrier
// waits on every CTA): 0 = plain launch (every CTA resident once the
// previous kernel ends, the grid being at most one CTA per SM), 1 =
// cooperative.  See ft_set_cooperative_quantizer.
std::atomic<int> g_qres_cooperative{0};

// GEMM tiling: 0 = CTA pairs whenever the activation has more than 128
// rows, 1 = one CTA per tile always.  See ft_set_gemm_mode.
std::atomic<int> g_gemm_mode{0};

// Launches k_qres with programmatic stream serialization; cooperative when
// requested and the kernel computes the tensor amax itself.
ft_status launch_qres(const ft::qres::Params& p, int mt, int splits, cudaStream_t st) {
    namespace Q = ft::qres;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)mt, (unsigned)splits, 1);
    cfg.blockDim = dim3(Q::NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = Q::make_layout(p.cchunk / Q::BKC, p.ring_bytes).total;
    cfg.stream = st;
    // it may start its setup while the previous kernel finishes (it waits
    // for that kernel's results on the device)
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (!p.amax_in && g_qres_cooperative.load(std::memory_order_relaxed)) ? 2 : 1;
    {
        LaunchTimer _lt(KID_QRES, st);
        FT_TRY(cuda_ok(cudaLaunchKernelEx(&cfg, Q::k_qres, p)));
        _lt.stop();
    }
    return last_launch();
}

// Q(T), g_T and P = [bf16(T L1) | bf16(s T L2)] for T [M, C], with the
// tensor amax computed on the way (amax_in == null) or taken from the caller.
// When the CTAs' chunks fit in shared memory all at once, one launch of
// k_qres reads T from HBM once; otherwise the amax pass (if needed) is
// followed by k_qdown (or the plain 1x16 quantizer when r == 0).
ft_status run_quant_down(const void* T, int64_t M, int64_t C, const void* L1, int64_t r1,
                         const void* L2, int64_t r2, float s, const float* amax_in, uint8_t* codes,
                         uint8_t* scales, float* tscale, void* P, uint8_t* ws, const WsPlan& w,
                         const DevInfo* d, cudaStream_t st, DepFlag* dep) {
    *dep = DepFlag();
    namespace Q = ft::qres;
    const int64_t r = r1 + r2;
    Q::Params p;
    std::memset(&p, 0, sizeof(p));
    p.do_mma = r > 0 ? 1 : 0;
    p.f1 = qres_factor(r1);
    p.f2 = qres_factor(r2);
    qres_ring(p);
    int mt = 0, splits = 0, cchunk = 0;
    if (!qres_grid(M, C, qres_max_stages(p.ring_bytes), d, &mt, &splits, &cchunk) || mt > QRES_MAX_ROW_TILES) {
        const float* a = amax_in;
        if (!a) {
            FT_TRY(run_amax(T, M, C, C, reinterpret_cast<float*>(ws + w.amax), d, st));
            a = reinterpret_cast<float*>(ws + w.amax);
        }
        return run_qdown(T, M, C, L1, r1, L2, r2, s, a, codes, scales, tscale, P, ws, w, d, st);
    }
    if (r1 > 0) FT_TRY(encode_factor_atoms(&p.mapL1, L1, C, r1));
    if (r2 > 0) FT_TRY(encode_factor_atoms(&p.mapL2, L2, C, r2));
    FT_TRY(encode_2d(&p.mapT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, T, C, M, C * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B));
    p.amax_in = amax_in;
    p.sync = reinterpret_cast<unsigned long long*>(ws + w.sync);
    p.epoch = next_epoch();
    p.tscale = tscale;
    p.codes = codes;
    p.scales = scales;
    p.slab = ws + w.sfslab;
    p.part = reinterpret_cast<float*>(ws + w.part);
    p.P = static_cast<__nv_bfloat16*>(P);
    p.counters = reinterpret_cast<unsigned long long*>(ws + w.qcnt);
    p.count_done = 1;
    p.M = (int)M;
    p.C = (int)C;
    p.r = (int)r;
    p.r1 = (int)r1;
    p.cchunk = cchunk;
    p.splits = splits;
    p.s = s;
    p.num_ctas = (unsigned)(mt * splits);
    FT_TRY(launch_qres(p, mt, splits, st));
    dep->done = p.sync + 2;
    dep->epoch = p.epoch;
    dep->count = p.num_ctas;
    return FT_OK;
}

// 1x16 quantization of a dense T [M, C] through the resident kernel (no
// down-projection) when it fits; sync: three epoch-tagged words (any content
// left by earlier calls).  Returns false in *done when the tensor does not fit.
ft_status run_quant_1x16_resident(const void* T, int64_t M, int64_t C, const float* amax_in,
                                  unsigned long long* sync, uint8_t* codes, uint8_t* scales,
                                  float* tscale, const DevInfo* d, cudaStream_t st, bool* done) {
    namespace Q = ft::qres;
    Q::Params p;
    std::memset(&p, 0, sizeof(p));
    qres_ring(p);
    int mt = 0, splits = 0, cchunk = 0;
    *done = false;
    if (!qres_grid(M, C, qres_max_stages(p.ring_bytes), d, &mt, &splits, &cchunk)) return FT_OK;
    *done = true;
    FT_TRY(encode_2d(&p.mapT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, T, C, M, C * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B));
    p.amax_in = amax_in;
    p.sync = sync;
    p.epoch = next_epoch();
    p.tscale = tscale;
    p.codes = codes;
    p.scales = scales;
    p.M = (int)M;
    p.C = (int)C;
    p.cchunk = cchunk;
    p.splits = splits;
    p.s = 1.0f;
    p.num_ctas = (unsigned)(mt * splits);
    return launch_qres(p, mt, splits, st);
}

// Panels of one low-rank factor in the GEMM: K-major, swizzled to the
// factor's width (16, 32 or 64 columns; two 64-wide atoms above 64).
ft::gemm::LrFactor gemm_factor(int64_t rf, int64_t pcol) {
    ft::gemm::LrFactor f;
    std::memset(&f, 0, sizeof(f));
    f.rf = (int)rf;
    f.pcol = (int)pcol;
    if (rf <= 0) return f;
    f.wbox = rf <= 16 ? 16 : rf <= 32 ? 32 : 64;
    f.natoms = rf <= 64 ? 1 : 2;
    f.swz = f.wbox == 16 ? ft::SWZ_32B : f.wbox == 32 ? ft::SWZ_64B : ft::SWZ_128B;
    f.row_bytes = (uint32_t)f.wbox * 2u;
    return f;
}

CUtensorMapSwizzle swizzle_for(int wbox) {
    return wbox == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : wbox == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                               : CU_TENSOR_MAP_SWIZZLE_128B;
}

// out[M, Nout] = ga gb Q(A) Q(B)^T + P[:, :r1] L1^T + P[:, r1:] L2^T, the
// block scales of A and B given as slabs ([rows/128][Kc/64][512]).  bf16:
// the 16-bit variant, out = gb A B^T + ..., with A = a_codes a bf16 [M, Kc]
// matrix and B = b_op the weight's bf16 image [Nout, Kc] (a_slab and ga
// unused).
// MLP fusion: the epilogue's GELU and the quantized copy of its output.
struct MlpOut {
    const float* amax_h;
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* slab;
    float* tscale;
};

ft_status run_gemm(bool bf16, const uint8_t* a_codes, const uint8_t* a_slab, const float* ga, int64_t M,
                   int64_t Kc, const uint8_t* b_op, const float* gb,
                   int64_t Nout, const void* P, const void* L1, int64_t r1, const void* L2, int64_t r2,
                   void* out, ft_dtype ot, const DevInfo* d, cudaStream_t st, DepFlag dep,
                   const MlpOut* mlp = nullptr, float* amax_out = nullptr) {
    Params p;
    std::memset(&p, 0, sizeof(p));
    p.amax_out = reinterpret_cast<unsigned int*>(amax_out);
    // CTA pairs for the 4-bit GEMM unless a tile's 128 rows hold every row
    const bool pair = !bf16 && M > ft::gemm::BM && g_gemm_mode.load(std::memory_order_relaxed) == 0;
    const int lrows = pair ? 64 : ft::gemm::BN;  // rows of an L panel box
    if (mlp) {
        p.mlp = 1;
        p.amax_h = mlp->amax_h;
        p.q_codes = mlp->codes;
        p.q_scales = mlp->scales;
        p.q_slab = mlp->slab;
        p.q_tscale = mlp->tscale;
    }
    if (bf16) {
        FT_TRY(encode_2d(&p.mapA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a_codes, Kc, M, Kc * 2, 64, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B));
        FT_TRY(encode_2d(&p.mapB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b_op, Kc, Nout, Kc * 2, 64, 256,
                         CU_TENSOR_MAP_SWIZZLE_128B));
    } else if (pair) {
        FT_TRY(encode_2d(&p.mapA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, Kc / 2, M, Kc / 2, 128, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B));
        // the weight's operand image as rows of 128 bytes, 288 per block
        // (256 code rows, 32 scale rows): one CTA's 128 code rows are one
        // box, the block's scale rows another
        const int64_t img_rows = (Nout / 256) * (Kc / 256) * ft::gemm::IMG_BLOCK_ROWS;
        FT_TRY(encode_2d(&p.mapB, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_op, 128, img_rows, 128, 128, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B));
        FT_TRY(encode_2d(&p.mapBs, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_op, 128, img_rows, 128, 128, 32,
                         CU_TENSOR_MAP_SWIZZLE_128B));
        FT_TRY(encode_slabs(&p.mapSFA, a_slab, Kc / 64, cdiv(M, 128), 1));
    } else {
        FT_TRY(encode_2d(&p.mapA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, Kc / 2, M, Kc / 2, 128, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B));
        // the weight's operand image (ft_pack_weight_operands) as a 3-D byte
        // tensor {128, 144, 2 * blocks}: one block (codes + scales of a
        // 256-row tile for one stage) is one box of {128, 144, 2}
        cuuint64_t dims[3] = {128, 144, (cuuint64_t)((Nout / 256) * (Kc / 256) * 2)};
        cuuint64_t strides[2] = {128, 144 * 128};
        cuuint32_t box[3] = {128, 144, 2};
        cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode(&p.mapB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(b_op), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return FT_ERR_CUDA;
        FT_TRY(encode_slabs(&p.mapSFA, a_slab, Kc / 64, cdiv(M, 128), 1));
    }
    const int64_t r = r1 + r2;
    p.f1 = gemm_factor(r1, 0);
    p.f2 = gemm_factor(r2, r1);
    if (r1 > 0) {
        FT_TRY(encode_2d(&p.mapP1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P, r, M, r * 2, p.f1.wbox, 128,
                         swizzle_for(p.f1.wbox)));
        FT_TRY(encode_2d(&p.mapL1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1, r1, Nout, r1 * 2, p.f1.wbox, lrows,
                         swizzle_for(p.f1.wbox)));
    }
    if (r2 > 0) {
        FT_TRY(encode_2d(&p.mapP2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P, r, M, r * 2, p.f2.wbox, 128,
                         swizzle_for(p.f2.wbox)));
        FT_TRY(encode_2d(&p.mapL2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2, r2, Nout, r2 * 2, p.f2.wbox, lrows,
                         swizzle_for(p.f2.wbox)));
    }
    p.out = static_cast<uint8_t*>(out);
    p.dep_done = dep.done;
    p.dep_epoch = dep.epoch;
    p.dep_count = dep.count;
    p.ga = bf16 ? nullptr : ga;
    p.gb = gb;
    p.out_f32 = (ot == FT_F32);
    p.M = (int)M;
    p.Nout = (int)Nout;
    p.Kc = (int)Kc;
    const int pr = pair ? 1 : 0;
    int stages = ft::gemm::MAX_STAGES;
    while (stages > 1 && ft::gemm::make_layout(stages, p.f1, p.f2, p.mlp, pr).total > 227u * 1024u) --stages;
    if (ft::gemm::make_layout(stages, p.f1, p.f2, p.mlp, pr).total > 227u * 1024u) return FT_ERR_SHAPE;
    p.stages = stages;
    const uint32_t smem = ft::gemm::make_layout(stages, p.f1, p.f2, p.mlp, pr).total;
    const int tiles = cdiv(M, pair ? 2 * ft::gemm::BM : ft::gemm::BM) * (int)(Nout / ft::gemm::BN);
    // persistent: one CTA (pair: two, one per SM of a TPC) per tile, at most
    // the device's SMs
    const int grid = pair ? 2 * std::max(1, std::min(tiles, d->sms / 2)) : std::max(1, std::min(tiles, d->sms));
    {
        LaunchTimer _lt(bf16 ? KID_GEMM_BF16 : KID_GEMM, st);
        const dim3 blk(ft::gemm::NUM_THREADS);
        if (bf16)
            FT_TRY(launch_overlapped(ft::gemm::k_gemm_fp4<true>, dim3((unsigned)grid), blk, smem, st, p));
        else if (pair && mlp)
            FT_TRY(launch_overlapped(ft::gemm::k_gemm_fp4<false, true, true>, dim3((unsigned)grid), blk, smem, st, p,
                                     2));
        else if (pair)
            FT_TRY(launch_overlapped(ft::gemm::k_gemm_fp4<false, false, true>, dim3((unsigned)grid), blk, smem, st,
                                     p, 2));
        else if (mlp)
            FT_TRY(launch_overlapped(ft::gemm::k_gemm_fp4<false, true>, dim3((unsigned)grid), blk, smem, st, p));
        else
            FT_TRY(launch_overlapped(ft::gemm::k_gemm_fp4<false>, dim3((unsigned)grid), blk, smem, st, p));
        _lt.stop();
    }
    return last_launch();
}

ft_status run_lora_grads(const void* dY, const void* X, const void* P, const void* Pg, int64_t M,
                         int64_t N, int64_t K, int64_t r_s, int64_t r_l, float* dA, float* dB,
                         uint8_t* ws, const WsPlan& w, const DevInfo* d, cudaStream_t st, DepFlag dep) {
    const int64_t r = r_s + r_l;
    ft::lgrad::Params p;
    std::memset(&p, 0, sizeof(p));
    namespace LG = ft::lgrad;
    FT_TRY(encode_colblocks(&p.mapT[0], dY, M, N, LG::BMR, 2));
    FT_TRY(encode_colblocks(&p.mapT[1], X, M, K, LG::BMR, 2));
    FT_TRY(encode_2d(&p.mapS[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P, r, M, r * 2, 64, LG::BMR,
                     CU_TENSOR_MAP_SWIZZLE_128B));
    FT_TRY(encode_2d(&p.mapS[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Pg, r, M, r * 2, 64, LG::BMR,
                     CU_TENSOR_MAP_SWIZZLE_128B));
    const int ctiles = (int)(N / ft::lgrad::BC + K / ft::lgrad::BC);
    int splits = std::max(1, std::min(LG_MAX_SPLITS, d->sms / std::max(1, ctiles)));
    int mrows = cdiv(M, (int64_t)splits * ft::lgrad::BMR) * ft::lgrad::BMR;
    splits = std::max(1, cdiv(M, mrows));
    float* partB = reinterpret_cast<float*>(ws + w.lgpart);
    float* partA = partB + (size_t)splits * N * r_l;
    p.part[0] = partB;
    p.part[1] = partA;
    p.out[0] = dB;
    p.out[1] = dA;
    p.counters = reinterpret_cast<unsigned long long*>(ws + w.lgcnt);
    p.epoch = next_epoch();
    p.C[0] = (int)N;
    p.C[1] = (int)K;
    p.M = (int)M;
    p.r_s = (int)r_s;
    p.r_l = (int)r_l;
    p.n_pad = r_l <= 64 ? 64 : 128;
    p.stages = LG::stages_for(p.n_pad);
    p.mrows = mrows;
    p.splits = splits;
    p.ctiles_max = LG_MAX_CTILES;
    p.dep_done = dep.done;
    p.dep_epoch = dep.epoch;
    p.dep_count = dep.count;
    dim3 grid((unsigned)(std::max(N, K) / ft::lgrad::BC), (unsigned)splits, 2);
    {
        LaunchTimer _lt(KID_LORA_GRAD, st);
        FT_TRY(launch_overlapped(ft::lgrad::k_lora_grad, grid, dim3(ft::lgrad::NUM_THREADS),
                                 ft::lgrad::smem_bytes(p.n_pad), st, p));
        _lt.stop();
    }
    return last_launch();
}

// ------------------------------------------------------------ validation
ft_status check_fp4_view(const ft_fp4* v, int64_t rows, int64_t cols, ft_block blk) {
    if (!v || !v->codes || !v->scales || !v->tscale) return FT_ERR_INVALID_ARG;
    if (v->rows != rows || v->cols != cols || v->blk != blk) return FT_ERR_SHAPE;
    if (!al16(v->codes) || !al16(v->scales) || (reinterpret_cast<uintptr_t>(v->tscale) & 3u))
        return FT_ERR_ALIGN;
    return FT_OK;
}

ft_status check_linear(const ft_linear* L) {
    if (!L) return FT_ERR_INVALID_ARG;
    if (L->N <= 0 || L->K <= 0 || L->r_s < 0 || L->r_l < 0) return FT_ERR_INVALID_ARG;
    if (L->N % 256 || L->K % 256) return FT_ERR_SHAPE;
    if (L->r_s % 16 || L->r_l % 16 || L->r_s + L->r_l > 128) return FT_ERR_SHAPE;
    if (L->N > (1 << 20) || L->K > (1 << 20)) return FT_ERR_SHAPE;
    if (L->w_k.blk == FT_BLK_1x16) {
        // 1x16 weight groups: two independent quantizations, W_res along K
        // and W_res^T along N, one tensor scale (read through w_k)
        FT_TRY(check_fp4_view(&L->w_k, L->N, L->K, FT_BLK_1x16));
        FT_TRY(check_fp4_view(&L->w_n, L->K, L->N, FT_BLK_1x16));
    } else {
        FT_TRY(check_fp4_view(&L->w_k, L->N, L->K, FT_BLK_16x16));
        if (!L->w_n.codes) return FT_ERR_INVALID_ARG;
        if (L->w_n.rows != L->K || L->w_n.cols != L->N || L->w_n.blk != FT_BLK_16x16) return FT_ERR_SHAPE;
        if (!al16(L->w_n.codes)) return FT_ERR_ALIGN;
        if ((L->w_n.scales && L->w_n.scales != L->w_k.scales) ||
            (L->w_n.tscale && L->w_n.tscale != L->w_k.tscale))
            return FT_ERR_INVALID_ARG;
    }
    if (L->r_s > 0 && (!L->U || !L->V)) return FT_ERR_INVALID_ARG;
    if (L->r_l > 0 && (!L->A || !L->B)) return FT_ERR_INVALID_ARG;
    if ((L->U && !al16(L->U)) || (L->V && !al16(L->V)) || (L->A && !al16(L->A)) ||
        (L->B && !al16(L->B)))
        return FT_ERR_ALIGN;
    if (!L->op_k || !L->op_n) return FT_ERR_INVALID_ARG;
    if (!al16(L->op_k) || !al16(L->op_n)) return FT_ERR_ALIGN;
    if (L->precision < FT_W4A4G4 || L->precision > FT_W4A16G16) return FT_ERR_INVALID_ARG;
    if ((L->precision & FT_W4A16G4) && !L->wd_k) return FT_ERR_INVALID_ARG;
    if ((L->precision & FT_W4A4G16) && !L->wd_n) return FT_ERR_INVALID_ARG;
    if ((L->wd_k && !al16(L->wd_k)) || (L->wd_n && !al16(L->wd_n))) return FT_ERR_ALIGN;
    return FT_OK;
}

}  // namespace

extern "C" {

const char* ft_status_str(ft_status s) {
    switch (s) {
        case FT_OK: return "FT_OK";
        case FT_ERR_INVALID_ARG: return "FT_ERR_INVALID_ARG";
        case FT_ERR_SHAPE: return "FT_ERR_SHAPE";
        case FT_ERR_ALIGN: return "FT_ERR_ALIGN";
        case FT_ERR_CUDA: return "FT_ERR_CUDA";
        case FT_ERR_TIMEOUT: return "FT_ERR_TIMEOUT";
        case FT_ERR_WORKSPACE: return "FT_ERR_WORKSPACE";
        case FT_ERR_UNSUPPORTED: return "FT_ERR_UNSUPPORTED";
    }
    return "FT_ERR_UNKNOWN";
}

size_t ft_quantize_workspace_bytes(void) { return 256; }

size_t ft_weight_operand_bytes(int64_t N, int64_t K) {
    if (N < 0 || K < 0) return 0;
    return (size_t)(N / 256) * (size_t)(K / 256) * 288u * 128u;
}

ft_status ft_pack_weight_operands(const uint8_t* codes_k, const uint8_t* codes_n, const uint8_t* grid,
                                  int64_t N, int64_t K, uint8_t* op_k, uint8_t* op_n, void* stream) {
    if (!codes_k || !codes_n || !grid || !op_k || !op_n || N < 0 || K < 0) return FT_ERR_INVALID_ARG;
    if (N % 256 || K % 256) return FT_ERR_SHAPE;
    if (!al16(codes_k) || !al16(codes_n) || !al16(op_k) || !al16(op_n)) return FT_ERR_ALIGN;
    if (N == 0 || K == 0) return FT_OK;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t chunks = (int64_t)ft_weight_operand_bytes(N, K) / 16;
    const int grid_n = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(chunks, 256), (int64_t)d->sms * 16));
    ft::k_pack_wop<<<grid_n, 256, 0, st>>>(codes_k, grid, nullptr, N, K, 0, op_k);
    FT_TRY(last_launch());
    ft::k_pack_wop<<<grid_n, 256, 0, st>>>(codes_n, grid, nullptr, N, K, 1, op_n);
    return last_launch();
}

ft_status ft_pack_weight_operands_1x16(const uint8_t* codes_k, const uint8_t* scales_k, const uint8_t* codes_n,
                                       const uint8_t* scales_n, int64_t N, int64_t K, uint8_t* op_k,
                                       uint8_t* op_n, void* stream) {
    if (!codes_k || !scales_k || !codes_n || !scales_n || !op_k || !op_n || N < 0 || K < 0)
        return FT_ERR_INVALID_ARG;
    if (N % 256 || K % 256) return FT_ERR_SHAPE;
    if (!al16(codes_k) || !al16(codes_n) || !al16(op_k) || !al16(op_n)) return FT_ERR_ALIGN;
    if (N == 0 || K == 0) return FT_OK;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t chunks = (int64_t)ft_weight_operand_bytes(N, K) / 16;
    const int grid_n = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(chunks, 256), (int64_t)d->sms * 16));
    ft::k_pack_wop<<<grid_n, 256, 0, st>>>(codes_k, nullptr, scales_k, N, K, 0, op_k);
    FT_TRY(last_launch());
    ft::k_pack_wop<<<grid_n, 256, 0, st>>>(codes_n, nullptr, scales_n, N, K, 1, op_n);
    return last_launch();
}

ft_status ft_dequant_weight_operands(const ft_fp4* w_k, const ft_fp4* w_n, void* wd_k, void* wd_n, void* stream) {
    if (!w_k || (!wd_k && !wd_n) || (wd_n && !w_n)) return FT_ERR_INVALID_ARG;
    const ft_block blk = w_k->blk;
    if (blk != FT_BLK_1x16 && blk != FT_BLK_16x16) return FT_ERR_INVALID_ARG;
    const int64_t N = w_k->rows, K = w_k->cols;
    if (N < 0 || K < 0) return FT_ERR_INVALID_ARG;
    if (N % 16 || K % 16) return FT_ERR_SHAPE;
    if (!w_k->codes || !w_k->scales) return FT_ERR_INVALID_ARG;
    if (wd_n) {
        if (!w_n->codes || w_n->blk != blk) return FT_ERR_INVALID_ARG;
        if (w_n->rows != K || w_n->cols != N) return FT_ERR_SHAPE;
        if (blk == FT_BLK_1x16 && !w_n->scales) return FT_ERR_INVALID_ARG;
        if (!al16(w_n->codes) || !al16(wd_n)) return FT_ERR_ALIGN;
    }
    if (!al16(w_k->codes) || (wd_k && !al16(wd_k))) return FT_ERR_ALIGN;
    if (N == 0 || K == 0) return FT_OK;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(N * K / 8, 256), (int64_t)d->sms * 16));
    if (wd_k) {
        LaunchTimer _lt(KID_DEQUANT_W, st);
        ft::k_dequant_w<<<grid, 256, 0, st>>>(w_k->codes, w_k->scales, N, K, blk == FT_BLK_16x16 ? 0 : 2,
                                              static_cast<uint16_t*>(wd_k));
        _lt.stop();
        FT_TRY(last_launch());
    }
    if (wd_n) {
        // 16x16: the codes packed along N with the one grid read transposed
        LaunchTimer _lt(KID_DEQUANT_W, st);
        ft::k_dequant_w<<<grid, 256, 0, st>>>(w_n->codes, blk == FT_BLK_16x16 ? w_k->scales : w_n->scales, K, N,
                                              blk == FT_BLK_16x16 ? 1 : 2, static_cast<uint16_t*>(wd_n));
        _lt.stop();
        FT_TRY(last_launch());
    }
    return FT_OK;
}

ft_status ft_gelu_bf16(const void* y, void* h, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (!y || !h))) return FT_ERR_INVALID_ARG;
    if (n % 8) return FT_ERR_SHAPE;
    if (!al16(y) || !al16(h)) return FT_ERR_ALIGN;
    if (n == 0) return FT_OK;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // one CTA of 1024 threads per SM: each CTA fills its own GELU table
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(n / 8, 1024), (int64_t)d->sms));
    LaunchTimer _lt(KID_GELU, st);
    ft::k_gelu_bf16<<<grid, 1024, 0, st>>>(static_cast<const uint16_t*>(y), static_cast<uint16_t*>(h), n);
    _lt.stop();
    return last_launch();
}

size_t ft_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r_s, int64_t r_l) {
    if (M < 0 || N < 0 || K < 0 || r_s < 0 || r_l < 0) return 0;
    return plan_ws(M, N, K, r_s, r_l).total;
}

ft_status ft_workspace_qact(int64_t M, int64_t N, int64_t K, int64_t r_s, int64_t r_l,
                            size_t* codes_off, size_t* scales_off, size_t* tscale_off) {
    if (M < 0 || N < 0 || K < 0 || r_s < 0 || r_l < 0) return FT_ERR_INVALID_ARG;
    if (!codes_off || !scales_off || !tscale_off) return FT_ERR_INVALID_ARG;
    const WsPlan w = plan_ws(M, N, K, r_s, r_l);
    *codes_off = w.codes;
    *scales_off = w.scales;
    *tscale_off = w.gact;
    return FT_OK;
}

ft_status ft_set_cooperative_quantizer(int on) {
    g_qres_cooperative.store(on ? 1 : 0, std::memory_order_relaxed);
    return FT_OK;
}

ft_status ft_set_gemm_mode(int mode) {
    if (mode != 0 && mode != 1) return FT_ERR_INVALID_ARG;
    g_gemm_mode.store(mode, std::memory_order_relaxed);
    return FT_OK;
}

ft_status ft_device_error(int* code, void* stream) {
    if (!code) return FT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int v = 0;
    FT_TRY(cuda_ok(cudaMemcpyFromSymbolAsync(&v, ft::g_ft_error, sizeof(int), 0,
                                             cudaMemcpyDeviceToHost, st)));
    FT_TRY(cuda_ok(cudaStreamSynchronize(st)));
    if (v) {
        const int zero = 0;
        FT_TRY(cuda_ok(cudaMemcpyToSymbolAsync(ft::g_ft_error, &zero, sizeof(int), 0,
                                               cudaMemcpyHostToDevice, st)));
        FT_TRY(cuda_ok(cudaStreamSynchronize(st)));
    }
    *code = v;
    return v ? FT_ERR_TIMEOUT : FT_OK;
}

ft_status ft_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, ft_block blk,
                      const float* amax, ft_fp4* out, void* ws, size_t ws_bytes, void* stream) {
    if (!x || !out) return FT_ERR_INVALID_ARG;
    if (blk != FT_BLK_1x16 && blk != FT_BLK_16x16) return FT_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return FT_ERR_INVALID_ARG;
    if (cols % 16 || (blk == FT_BLK_16x16 && rows % 16)) return FT_ERR_SHAPE;
    FT_TRY(check_fp4_view(out, rows, cols, blk));
    if (!al16(x) || (ld % 8)) return FT_ERR_ALIGN;
    if (!amax && (!ws || ws_bytes < ft_quantize_workspace_bytes())) return FT_ERR_WORKSPACE;
    if (amax && (reinterpret_cast<uintptr_t>(amax) & 3u)) return FT_ERR_ALIGN;
    if (rows == 0 || cols == 0) return FT_OK;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (blk == FT_BLK_1x16 && ld == cols) {
        bool done = false;
        // the amax slot sits at the start of the workspace, the
        // synchronisation words 64 bytes in
        unsigned long long* sync = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(ws) + 64);
        FT_TRY(run_quant_1x16_resident(x, rows, cols, amax, sync, out->codes,
                                       out->scales, out->tscale, d, st, &done));
        if (done) return FT_OK;
    }
    const float* a = amax;
    if (!a) {
        float* slot = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 128);
        FT_TRY(run_amax(x, rows, cols, ld, slot, d, st));
        a = slot;
    }
    if (blk == FT_BLK_1x16)
        return run_quant_1x16(x, rows, cols, ld, a, out->codes, out->scales, out->tscale, nullptr, d, st);
    return run_tile16(true, x, rows, cols, ld, a, out->codes, out->scales, nullptr, nullptr,
                      out->tscale, nullptr, d, st);
}

ft_status ft_quantize_transpose(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                ft_block blk, const float* amax, ft_fp4* out_row, ft_fp4* out_col,
                                void* ws, size_t ws_bytes, void* stream) {
    if (!x || !out_row || !out_col) return FT_ERR_INVALID_ARG;
    if (blk != FT_BLK_1x16 && blk != FT_BLK_16x16) return FT_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return FT_ERR_INVALID_ARG;
    if (rows % 16 || cols % 16) return FT_ERR_SHAPE;
    FT_TRY(check_fp4_view(out_row, rows, cols, blk));
    if (!out_col->codes) return FT_ERR_INVALID_ARG;
    if (out_col->rows != cols || out_col->cols != rows || out_col->blk != blk) return FT_ERR_SHAPE;
    if (!al16(out_col->codes)) return FT_ERR_ALIGN;
    if (blk == FT_BLK_16x16) {
        if ((out_col->scales && out_col->scales != out_row->scales) ||
            (out_col->tscale && out_col->tscale != out_row->tscale))
            return FT_ERR_INVALID_ARG;
    } else {
        if (!out_col->scales || !out_col->tscale) return FT_ERR_INVALID_ARG;
        if (!al16(out_col->scales) || (reinterpret_cast<uintptr_t>(out_col->tscale) & 3u))
            return FT_ERR_ALIGN;
    }
    if (!al16(x) || (ld % 8)) return FT_ERR_ALIGN;
    if (!amax && (!ws || ws_bytes < ft_quantize_workspace_bytes())) return FT_ERR_WORKSPACE;
    if (rows == 0 || cols == 0) return FT_OK;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float* a = amax;
    if (!a) {
        float* slot = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 128);
        FT_TRY(run_amax(x, rows, cols, ld, slot, d, st));
        a = slot;
    }
    if (blk == FT_BLK_16x16)
        return run_tile16(true, x, rows, cols, ld, a, out_row->codes, out_row->scales,
                          out_col->codes, nullptr, out_row->tscale, nullptr, d, st);
    return run_tile16(false, x, rows, cols, ld, a, out_row->codes, out_row->scales, out_col->codes,
                      out_col->scales, out_row->tscale,
                      out_col->tscale != out_row->tscale ? out_col->tscale : nullptr, d, st);
}

ft_status ft_linear_fwd(const ft_linear* L, const void* X, int64_t M, const float* amax_x, void* Y,
                        ft_dtype yt, void* P_save, float* amax_y, void* ws, size_t ws_bytes, void* stream) {
    FT_TRY(check_linear(L));
    if (M < 0) return FT_ERR_INVALID_ARG;
    if (yt != FT_BF16 && yt != FT_F32) return FT_ERR_INVALID_ARG;
    if (M > (1 << 24)) return FT_ERR_SHAPE;
    const int64_t r = L->r_s + L->r_l;
    if (M == 0) return FT_OK;
    if (!X || !Y || (r > 0 && !P_save)) return FT_ERR_INVALID_ARG;
    if (!al16(X) || !al16(Y) || (P_save && !al16(P_save)) || (reinterpret_cast<uintptr_t>(amax_y) & 3u))
        return FT_ERR_ALIGN;
    const WsPlan w = plan_ws(M, L->N, L->K, L->r_s, L->r_l);
    if (!ws || ws_bytes < w.total || !al16(ws)) return FT_ERR_WORKSPACE;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    float* g_x = reinterpret_cast<float*>(wsb + w.gact);
    uint8_t* codes = wsb + w.codes;
    uint8_t* scales = wsb + w.scales;
    DepFlag dep;
    FT_TRY(run_quant_down(X, M, L->K, L->U, L->r_s, L->A, L->r_l, L->s, amax_x, codes, scales, g_x,
                          P_save, wsb, w, d, st, &dep));
    if (L->precision & FT_W4A16G4)  // 16-bit activations: the GEMM reads X itself
        return run_gemm(true, static_cast<const uint8_t*>(X), nullptr, nullptr, M, L->K,
                        static_cast<const uint8_t*>(L->wd_k), L->w_k.tscale, L->N, P_save, L->V, L->r_s, L->B,
                        L->r_l, Y, yt, d, st, dep, nullptr, amax_y);
    return run_gemm(false, codes, wsb + w.sfslab, g_x, M, L->K, L->op_k, L->w_k.tscale, L->N,
                    P_save, L->V, L->r_s, L->B, L->r_l, Y, yt, d, st, dep, nullptr, amax_y);
}

ft_status ft_linear_bwd(const ft_linear* L, const void* dY, const void* X, const void* P_save,
                        int64_t M, const float* amax_dy, void* dX, ft_dtype xt, float* dA,
                        float* dB, void* ws, size_t ws_bytes, void* stream) {
    FT_TRY(check_linear(L));
    if (M < 0) return FT_ERR_INVALID_ARG;
    if (xt != FT_BF16 && xt != FT_F32) return FT_ERR_INVALID_ARG;
    if (M > (1 << 24)) return FT_ERR_SHAPE;
    const int64_t r = L->r_s + L->r_l;
    if (L->r_l > 0 && (!dA || !dB)) return FT_ERR_INVALID_ARG;
    if ((dA && !al16(dA)) || (dB && !al16(dB))) return FT_ERR_ALIGN;
    if (M == 0) {
        // no tokens: dX is empty and the adapter gradients are exactly zero
        if (L->r_l > 0) {
            DevInfo* d0;
            FT_TRY(device_info(&d0));
            cudaStream_t st0 = static_cast<cudaStream_t>(stream);
            FT_TRY(cuda_ok(cudaMemsetAsync(dA, 0, (size_t)L->K * L->r_l * 4, st0)));
            FT_TRY(cuda_ok(cudaMemsetAsync(dB, 0, (size_t)L->N * L->r_l * 4, st0)));
        }
        return FT_OK;
    }
    if (!dY || !dX || (r > 0 && !P_save) || (L->r_l > 0 && !X)) return FT_ERR_INVALID_ARG;
    if (!al16(dY) || !al16(dX) || (X && !al16(X)) || (P_save && !al16(P_save))) return FT_ERR_ALIGN;
    const WsPlan w = plan_ws(M, L->N, L->K, L->r_s, L->r_l);
    if (!ws || ws_bytes < w.total || !al16(ws)) return FT_ERR_WORKSPACE;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    float* g_dy = reinterpret_cast<float*>(wsb + w.gact);
    uint8_t* codes = wsb + w.codes;
    uint8_t* scales = wsb + w.scales;
    void* Pg = wsb + w.pg;
    DepFlag dep;
    FT_TRY(run_quant_down(dY, M, L->N, L->V, L->r_s, L->B, L->r_l, L->s, amax_dy, codes, scales, g_dy,
                          Pg, wsb, w, d, st, &dep));
    if (L->precision & FT_W4A4G16)  // 16-bit gradients: the dgrad GEMM reads dY itself
        FT_TRY(run_gemm(true, static_cast<const uint8_t*>(dY), nullptr, nullptr, M, L->N,
                        static_cast<const uint8_t*>(L->wd_n), L->w_k.tscale, L->K, Pg, L->U, L->r_s, L->A, L->r_l,
                        dX, xt, d, st, dep));
    else
        FT_TRY(run_gemm(false, codes, wsb + w.sfslab, g_dy, M, L->N, L->op_n, L->w_k.tscale, L->K,
                        Pg, L->U, L->r_s, L->A, L->r_l, dX, xt, d, st, dep));
    // the adapter gradients read dY, X, P_save and Pg: nothing the dgrad GEMM
    // (the kernel they overlap) writes, so they wait on the quantizer's
    // counter for Pg, not on the GEMM
    if (L->r_l > 0)
        FT_TRY(run_lora_grads(dY, X, P_save, Pg, M, L->N, L->K, L->r_s, L->r_l, dA, dB, wsb, w, d, st, dep));
    return FT_OK;
}

size_t ft_mlp_workspace_bytes(const ft_linear* up, const ft_linear* down, int64_t M) {
    if (!up || !down || M < 0) return 0;
    return up256(plan_ws(M, up->N, up->K, up->r_s, up->r_l).total) +
           plan_ws(M, down->N, down->K, down->r_s, down->r_l).total;
}

ft_status ft_mlp_fwd(const ft_linear* up, const ft_linear* down, const void* X, int64_t M, const float* amax_x,
                     const float* amax_h, void* H, void* Y, ft_dtype yt, void* P_up, void* P_down, float* amax_h_out,
                     void* ws, size_t ws_bytes, void* stream) {
    FT_TRY(check_linear(up));
    FT_TRY(check_linear(down));
    if (down->K != up->N) return FT_ERR_SHAPE;
    if (up->precision != FT_W4A4G4 || down->precision != FT_W4A4G4) return FT_ERR_INVALID_ARG;
    if (M < 0) return FT_ERR_INVALID_ARG;
    if (yt != FT_BF16 && yt != FT_F32) return FT_ERR_INVALID_ARG;
    if (M > (1 << 24)) return FT_ERR_SHAPE;
    if (M == 0) return FT_OK;
    const int64_t r_up = up->r_s + up->r_l, r_dn = down->r_s + down->r_l;
    if (!X || !amax_h || !H || !Y || (r_up > 0 && !P_up) || (r_dn > 0 && !P_down)) return FT_ERR_INVALID_ARG;
    // H leaves the fused epilogue in whole 32-byte sectors
    if (!al16(X) || (reinterpret_cast<uintptr_t>(H) & 31u) || !al16(Y) || (P_up && !al16(P_up)) ||
        (P_down && !al16(P_down)) || (reinterpret_cast<uintptr_t>(amax_h) & 3u) ||
        (reinterpret_cast<uintptr_t>(amax_h_out) & 3u))
        return FT_ERR_ALIGN;
    const WsPlan wu = plan_ws(M, up->N, up->K, up->r_s, up->r_l);
    const WsPlan wd = plan_ws(M, down->N, down->K, down->r_s, down->r_l);
    if (!ws || ws_bytes < up256(wu.total) + wd.total || !al16(ws)) return FT_ERR_WORKSPACE;
    DevInfo* d;
    FT_TRY(device_info(&d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* wsu = static_cast<uint8_t*>(ws);
    uint8_t* wsd = wsu + up256(wu.total);
    // FC1: Q(X) and P_up in one pass over X
    DepFlag dep;
    FT_TRY(run_quant_down(X, M, up->K, up->U, up->r_s, up->A, up->r_l, up->s, amax_x, wsu + wu.codes,
                          wsu + wu.scales, reinterpret_cast<float*>(wsu + wu.gact), P_up, wsu, wu, d, st, &dep));
    // FC1's GEMM with the fused epilogue: H = GELU(bf16(Y_up)) and Q(H) in
    // the down layer's workspace, as its own quantizer would lay it out
    MlpOut mo;
    mo.amax_h = amax_h;
    mo.codes = wsd + wd.codes;
    mo.scales = wsd + wd.scales;
    mo.slab = wsd + wd.sfslab;
    mo.tscale = reinterpret_cast<float*>(wsd + wd.gact);
    FT_TRY(run_gemm(false, wsu + wu.codes, wsu + wu.sfslab, reinterpret_cast<float*>(wsu + wu.gact), M, up->K,
                    up->op_k, up->w_k.tscale, up->N, P_up, up->V, up->r_s, up->B, up->r_l, H, FT_BF16, d, st, dep,
                    &mo, amax_h_out));
    // FC2: its down-projections of H (no second quantization), then its GEMM on Q(H)
    FT_TRY(run_qdown(H, M, down->K, down->U, down->r_s, down->A, down->r_l, down->s, nullptr, nullptr, nullptr,
                     nullptr, P_down, wsd, wd, d, st, false));
    return run_gemm(false, wsd + wd.codes, wsd + wd.sfslab, reinterpret_cast<float*>(wsd + wd.gact), M, down->K,
                    down->op_k, down->w_k.tscale, down->N, P_down, down->V, down->r_s, down->B, down->r_l, Y, yt, d,
                    st, DepFlag());
}

ft_status ft_timing_enable(int on) {
    std::lock_guard<std::mutex> lk(g_timing.mu);
    g_timing.on = on != 0;
    return FT_OK;
}

ft_status ft_timing_read(const char* kernel, double* total_ms, int64_t* launches) {
    if (!kernel || !total_ms || !launches) return FT_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_timing.mu);
    for (auto& r : g_timing.recs) {
        float ms = 0.0f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            return FT_ERR_CUDA;
        g_timing.ms[r.kid] += ms;
        g_timing.launches[r.kid] += 1;
        g_timing.pool.push_back(r.a);
        g_timing.pool.push_back(r.b);
    }
    g_timing.recs.clear();
    for (int k = 0; k < KID_COUNT; ++k)
        if (std::strcmp(kernel, kKernelNames[k]) == 0) {
            *total_ms = g_timing.ms[k];
            *launches = g_timing.launches[k];
            return FT_OK;
        }
    if (std::strcmp(kernel, "*") == 0) {
        double t = 0.0;
        int64_t n = 0;
        for (int k = 0; k < KID_COUNT; ++k) {
            t += g_timing.ms[k];
            n += g_timing.launches[k];
        }
        *total_ms = t;
        *launches = n;
        return FT_OK;
    }
    return FT_ERR_INVALID_ARG;
}

ft_status ft_timing_reset(void) {
    std::lock_guard<std::mutex> lk(g_timing.mu);
    for (auto& r : g_timing.recs) {
        cudaEventSynchronize(r.b);
        g_timing.pool.push_back(r.a);
        g_timing.pool.push_back(r.b);
    }
    g_timing.recs.clear();
    for (int k = 0; k < KID_COUNT; ++k) {
        g_timing.ms[k] = 0.0;
        g_timing.launches[k] = 0;
    }
    return FT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- forward without allocation
// Some callers cannot hand the library a workspace: a C host that has no
// device allocator wired in, a plug-in living inside another framework that
// owns all device memory through its own pool and forbids cudaMalloc from
// third-party code, or code that must not allocate while it builds up work
// on a stream.  ft_linear_fwd_noalloc serves them: it runs the same forward
// as ft_linear_fwd with its workspace in the array below, which lives in the
// library's device image.  Every GPU that loads the library holds these
// bytes until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_scratch_dev[64] = {};
unsigned long long g_noalloc_ctx[64] = {};

// Device address of g_noalloc_scratch on the current device.  The host
// symbol is only a stand-in; the address has to be looked up, once per
// device, with that device current -- and again after cudaDeviceReset, whose
// new context loads the library's device image (and the array) anew.  A
// fresh image holds the array zero-filled, as the calls' synchronisation
// words need.
ft_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    unsigned long long ctx = 0;
    FT_TRY(current_ctx_id(dev, &ctx));
    if (!g_noalloc_scratch_dev[dev] || g_noalloc_ctx[dev] != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FT_ERR_CUDA;
        g_noalloc_scratch_dev[dev] = p;
        g_noalloc_ctx[dev] = ctx;
    }
    *out = g_noalloc_scratch_dev[dev];
    return FT_OK;
}

}  // namespace

extern "C" ft_status ft_linear_fwd_noalloc(const ft_linear* L, const void* X, int64_t M,
                                           const float* amax_x, void* Y, ft_dtype yt, void* P_save,
                                           void* stream) {
    if (!L || M < 0 || L->N < 0 || L->K < 0 || L->r_s < 0 || L->r_l < 0) return FT_ERR_INVALID_ARG;
    if (ft_workspace_bytes(M, L->N, L->K, L->r_s, L->r_l) > kNoAllocScratchBytes) return FT_ERR_WORKSPACE;
    void* scratch = nullptr;
    FT_TRY(noalloc_scratch(&scratch));
    return ft_linear_fwd(L, X, M, amax_x, Y, yt, P_save, nullptr, scratch, kNoAllocScratchBytes, stream);
}

extern "C" size_t ft_linear_fwd_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }
