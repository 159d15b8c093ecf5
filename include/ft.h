/*
 * ft.h -- C ABI of the B200 (sm_100a) W4A4G4 triple-branch linear layer.
 *
 * The method is FourTune ("FourTune: Towards Fully 4-Bit Efficient
 * Post-Training for Diffusion Models"): every linear layer of a diffusion
 * transformer is split into three branches that read the same input and whose
 * outputs are summed (section 3.1, Eq. 2):
 *
 *     Y  = GEMM4(Q(X), Q(W_res))  +  (X U) V^T  +  s (X A) B^T
 *          frozen 4-bit backbone     frozen        trainable LoRA
 *                                    stabilizer
 *
 * and the backward pass propagates through all three (section 3.2, Eq. 3):
 *
 *     dX = GEMM4(Q(dY), Q(W_res)^T) + (dY V) U^T + s (dY B) A^T
 *     dB = s dY^T (X A)          dA = s X^T (dY B)
 *
 * Notation (PyTorch convention, weights stored [out, in]):
 *   X  [M, K] bf16      W_res [N, K] (the SVD residual of the weight, Eq. 1)
 *   U  [K, r_s] bf16    V [N, r_s] bf16   (V U^T = the top-r_s SVD part of W)
 *   A  [K, r_l] bf16    B [N, r_l] bf16   (the adapter; s its scale)
 *
 * Q() is NVFP4 block quantization: E2M1 4-bit codes, one E4M3 scale per
 * block, one FP32 tensor scale g.  Activations and gradients use 1x16 blocks
 * along the contiguous axis; weights use 16x16 blocks so that Q(W_res)^T is
 * the same codes read transposed with the same scale grid (section 3.2,
 * "block-wise quantization ... efficient online transposition").  Encoding,
 * with IEEE FP32 round-to-nearest-even at every step:
 *     g   = amax(tensor) / 2688          (g = 1 for an all-zero tensor)
 *     sd  = E4M3_rne_satfinite(amax(block) / (6 g))
 *     code= E2M1_rne_satfinite(x / (sd g)),  sign kept; code 0 when sd == 0
 *     deq = e2m1(code) * sd * g
 * Two codes per byte, the lower-index element in the low nibble.
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless stated; the caller owns every
 *     buffer (inputs, outputs, workspace).  The library never allocates.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Arguments are validated on the host
 *     first: on any FT_ERR_* return nothing has been launched.
 *   - bf16 matrices are row-major with a leading dimension in elements.
 *     Device pointers of bf16 inputs and of code/scale outputs must be 16-byte
 *     aligned and leading dimensions must keep rows 16-byte aligned
 *     (FT_ERR_ALIGN otherwise).
 *   - Empty inputs (zero rows) return FT_OK and launch nothing.
 *   - NaN or Inf inputs are outside the contract; results are unspecified.
 *   - Device-side failures (a bounded wait inside a kernel that ran out) set a
 *     device error word; read and clear it with ft_device_error().
 *   - Calls on one stream may be enqueued back to back without host
 *     synchronisation: each kernel completes only after every kernel before
 *     it on the stream, so a later call (or the caller's own kernel) never
 *     overwrites or reads a buffer an earlier call still uses.
 *   - The kernels of ft_quantize, ft_quantize_transpose (1x16, computed
 *     amax), ft_linear_fwd and ft_linear_bwd synchronise through counter
 *     words in the workspace, tagged with an epoch the host draws afresh for
 *     every call and writes into the launch's parameters.  Replaying a CUDA
 *     graph that captured such a call reuses its epochs: the counters
 *     already hold their final values from the previous replay, so the
 *     device waits would pass without waiting.  Do not replay captured calls.
 *   - The library caches per-device state (kernel attributes, module
 *     addresses) on first use and sets it up again in a new context of the
 *     device (after cudaDeviceReset); workspaces allocated in the old
 *     context are gone with it.
 */
#ifndef FT_H_
#define FT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FT_OK = 0,
    FT_ERR_INVALID_ARG = 1, /* null pointer, bad enum, negative size          */
    FT_ERR_SHAPE = 2,       /* a size is not a supported multiple             */
    FT_ERR_ALIGN = 3,       /* pointer or leading dimension misaligned        */
    FT_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed            */
    FT_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out (device word)  */
    FT_ERR_WORKSPACE = 6,   /* workspace missing or smaller than required     */
    FT_ERR_UNSUPPORTED = 7  /* the current device is not sm_100               */
} ft_status;

typedef enum { FT_BLK_1x16 = 0, FT_BLK_16x16 = 1 } ft_block;
typedef enum { FT_BF16 = 0, FT_F32 = 1 } ft_dtype;

/* Precision configuration of a layer (section 4, "Impact of Precision
 * Configurations", Table 4).  The weight is always 4-bit.  FT_W4A4G4 (the
 * method): both backbone GEMMs are NVFP4 x NVFP4.  Bit 0 (FT_W4A16G4): the
 * forward GEMM reads the bf16 activation X with the weight's bf16 image
 * (ft_linear.wd_k).  Bit 1 (FT_W4A4G16): the dgrad GEMM reads the bf16
 * output gradient dY with the transposed image (wd_n).  FT_W4A16G16: both.
 * The 16-bit GEMMs run on tcgen05 kind::f16 with FP32 accumulation; the
 * low-rank branches and the adapter gradients are the same in every
 * configuration (they never read a quantized tensor).                      */
typedef enum { FT_W4A4G4 = 0, FT_W4A16G4 = 1, FT_W4A4G16 = 2, FT_W4A16G16 = 3 } ft_precision;

/* Non-owning view of an NVFP4 tensor of logical shape rows x cols.
 *   codes : rows x cols/2 bytes, row-major, two E2M1 codes per byte packed
 *           along the row (column 2i in the low nibble of byte i).
 *   scales: E4M3 bytes, row-major.  FT_BLK_1x16: rows x cols/16 (one per 16
 *           consecutive elements of a row).  FT_BLK_16x16: rows/16 x cols/16.
 *   tscale: one float, the decode tensor scale g.                          */
typedef struct {
    uint8_t* codes;
    uint8_t* scales;
    float* tscale;
    int64_t rows;
    int64_t cols;
    ft_block blk;
} ft_fp4;

/* Non-owning description of one triple-branch linear layer (Eq. 2).
 *   w_k : Q(W_res), FT_BLK_16x16, rows = N, cols = K (codes packed along K).
 *   w_n : the same codes transposed, rows = K, cols = N (codes packed along
 *         N).  Its scales/tscale pointers must equal w_k's: one scale grid
 *         [N/16, K/16] serves both layouts (section 3.2).
 *   Or, for the granularity ablation (section 4, "Impact of Quantization
 *   Granularity", Table 5), both FT_BLK_1x16: w_k = Q(W_res) in 1x16 groups
 *   along K (scales [N, K/16]), w_n = Q(W_res^T), an independent 1x16
 *   quantization along N (scales [K, N/16]), as ft_quantize_transpose
 *   writes them; the tensor scale is read through w_k.
 *   U [K, r_s], V [N, r_s], A [K, r_l], B [N, r_l]: bf16, row-major, dense.
 *   r_s, r_l: multiples of 16 with r_s + r_l <= 128 (either may be 0).
 *   s: the LoRA scale.
 *   op_k, op_n: the 4-bit GEMMs' images of w_k and of w_n: codes and
 *         scales of each 256 x 256 block side by side, the scales one per
 *         row (ft_pack_weight_operands fills them from w_k, w_n and the
 *         grid; ft_weight_operand_bytes(N, K) bytes each, 16-byte aligned).
 *         A layout of the same codes and scales, not a new quantization.
 *   precision: an ft_precision (0 = FT_W4A4G4, the method).
 *   wd_k, wd_n: the weight's bf16 images for the 16-bit GEMMs
 *         (ft_dequant_weight_operands): wd_k [N, K] read by the forward
 *         when precision has FT_W4A16G4, wd_n [K, N] (the same values
 *         transposed) read by dgrad when it has FT_W4A4G16; NULL otherwise.
 *         16-byte aligned.                                                 */
typedef struct {
    int64_t N, K, r_s, r_l;
    float s;
    ft_fp4 w_k;
    ft_fp4 w_n;
    const void* U;
    const void* V;
    const void* A;
    const void* B;
    const uint8_t* op_k;
    const uint8_t* op_n;
    int32_t precision;
    const void* wd_k;
    const void* wd_n;
} ft_linear;

/* ft_quantize -- Q(x) for a bf16 matrix (section 3.2 block quantization).
 *   x     : bf16 [rows, cols], leading dimension ld (elements, ld >= cols).
 *   blk   : FT_BLK_1x16 (cols % 16 == 0) or FT_BLK_16x16 (rows % 16 == 0 and
 *           cols % 16 == 0).
 *   amax  : device float holding max|x| to use for the tensor scale, or NULL
 *           to compute it (needs ws_bytes >= ft_quantize_workspace_bytes()).
 *   out   : out->codes / scales / tscale receive the result; out->rows,
 *           out->cols and out->blk must equal rows, cols, blk.
 * Codes and scales match the encoding above bit for bit.                   */
ft_status ft_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, ft_block blk,
                      const float* amax, ft_fp4* out, void* ws, size_t ws_bytes, void* stream);

/* ft_quantize_transpose -- both layouts in one pass over x.
 *   FT_BLK_16x16: out_row = codes packed along rows of x ([rows, cols/2]);
 *     out_col = the same codes transposed ([cols, rows/2]); one scale grid
 *     [rows/16, cols/16] and one tensor scale, written through out_row
 *     (out_col->scales / tscale must be equal to out_row's or NULL).
 *   FT_BLK_1x16: out_row = Q(x) with blocks along rows; out_col = Q(x^T),
 *     an independent 1x16 quantization of the columns of x (blocks of 16
 *     consecutive rows), codes [cols, rows/2], scales [cols, rows/16].  Both
 *     share the tensor scale of x (written to both tscale pointers).
 *     Needs rows % 16 == 0 and cols % 16 == 0.                             */
ft_status ft_quantize_transpose(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                ft_block blk, const float* amax, ft_fp4* out_row,
                                ft_fp4* out_col, void* ws, size_t ws_bytes, void* stream);

/* ft_pack_weight_operands -- once per weight, after its 16x16 quantization:
 * writes the operand images the 4-bit GEMMs read, one per orientation
 * (section 3.2: the grid of a 16x16 block serves W_res and W_res^T alike,
 * so each grid entry is repeated for the 16 rows of its block in either
 * orientation; no value changes).
 *   codes_k : w_k.codes [N, K/2];  codes_n : w_n.codes [K, N/2].
 *   grid    : the [N/16, K/16] E4M3 scale grid of Q(W_res) (w_k.scales).
 *   op_k, op_n: ft_weight_operand_bytes(N, K) bytes each, 16-byte aligned.
 *   N, K    : multiples of 256.
 * Layout (an operand of R rows and C contraction columns): for each 256-row
 * tile t and 256-deep stage kt, a block of 288 rows of 128 bytes: rows
 * 0-255 = the codes of rows 256 t .. + 255, contraction bytes 128 kt ..
 * + 127; rows 256-287 = their scales for the stage, as two 128-row halves x
 * four 64-deep steps x 512 bytes, byte 16 l + 4 i + b of a step holding the
 * scale of half-row 32 i + l, columns 64 s + 16 b .. + 15 (the order
 * tcgen05.cp copies into the tensor memory's scale-factor layout), with
 * 16-byte chunk c of scale row p stored at chunk c ^ (p % 8) (undone by the
 * 128-byte swizzle of the copy that loads a block).  Blocks are ordered
 * (t, kt) with kt fastest.                                                 */
size_t ft_weight_operand_bytes(int64_t N, int64_t K);
ft_status ft_pack_weight_operands(const uint8_t* codes_k, const uint8_t* codes_n, const uint8_t* grid,
                                  int64_t N, int64_t K, uint8_t* op_k, uint8_t* op_n, void* stream);

/* ft_pack_weight_operands_1x16 -- the same images for 1x16 weight groups:
 * each operand's row-major scales (scales_k = w_k.scales [N, K/16] for
 * op_k, scales_n = w_n.scales [K, N/16] for op_n) take the grid's place,
 * one scale per row and 16 contraction columns already.  Arguments and
 * errors otherwise as ft_pack_weight_operands.                             */
ft_status ft_pack_weight_operands_1x16(const uint8_t* codes_k, const uint8_t* scales_k, const uint8_t* codes_n,
                                       const uint8_t* scales_n, int64_t N, int64_t K, uint8_t* op_k,
                                       uint8_t* op_n, void* stream);

/* ft_dequant_weight_operands -- once per weight, for the 16-bit GEMMs of
 * the precision configurations (section 4, Table 4): bf16 images of Q(W_res)
 * holding e2m1(code) x block scale (exact in bf16; the tensor scale stays in
 * w_k.tscale and is applied by the GEMM).  A layout of the same quantized
 * values, not a new quantization.
 *   w_k   : Q(W_res) [N, K] as in ft_linear (16x16 blocks, or 1x16 groups).
 *   w_n   : its dgrad orientation [K, N] (needed when wd_n is given; for
 *           16x16 blocks its scales are w_k's grid).
 *   wd_k  : bf16 [N, K] out, or NULL.   wd_n : bf16 [K, N] out, or NULL.
 *   N, K multiples of 16; 16-byte aligned pointers.  At least one output.  */
ft_status ft_dequant_weight_operands(const ft_fp4* w_k, const ft_fp4* w_n, void* wd_k, void* wd_n, void* stream);

/* ft_gelu_bf16 -- h = GELU(y) = y Phi(y) elementwise on bf16, each result
 * the correctly rounded bf16 of the exact GELU (round to nearest even): the
 * activation the fused MLP applies between its linears (section 3.3, "MLP
 * Fusion"), for callers that apply it outside the fused path.
 *   y, h : bf16 [n] device pointers, 16-byte aligned (may be equal); n a
 *          multiple of 8.  NaN inputs are outside the contract.            */
ft_status ft_gelu_bf16(const void* y, void* h, int64_t n, void* stream);

/* ft_linear_fwd -- Eq. 2 with LoRA fusion (section 3.3): one pass over X
 * emits Q(X) and the down-projections P = [bf16(X U) | bf16(s X A)]; one
 * FP4 GEMM on tcgen05 block-scaled tensor cores adds P [V | B]^T in its
 * epilogue and writes Y once.
 *   X      : bf16 [M, K] dense (ld = K).  M >= 0, any value.
 *   amax_x : device float max|X|, or NULL to compute it.
 *   Y      : [M, N] dense, FT_BF16 or FT_F32 (yt).
 *   P_save : bf16 [M, r_s + r_l] dense, written; the backward reads it.
 *   amax_y : NULL, or a device float >= 0 that the call raises to
 *            max(*amax_y, max|Y|) over Y as stored: the tensor amax of the
 *            next layer's input, found by the GEMM's epilogue without
 *            another pass over Y (section 3.3's fusion, the amax for a
 *            single-pass quantize next).  Zero it before the call to get
 *            max|Y| itself.  4-byte aligned (FT_ERR_ALIGN otherwise).
 *   N, K   : multiples of 256 (the scale rows stay 16-byte aligned for TMA).
 *   ws     : at least ft_workspace_bytes(M, N, K, r_s, r_l) bytes.         */
ft_status ft_linear_fwd(const ft_linear* L, const void* X, int64_t M, const float* amax_x,
                        void* Y, ft_dtype yt, void* P_save, float* amax_y, void* ws, size_t ws_bytes,
                        void* stream);

/* ft_linear_bwd -- Eq. 3 and the adapter gradients (section 3.2).
 *   dY      : bf16 [M, N] dense; X: the forward's bf16 [M, K];
 *   P_save  : the forward's P.
 *   amax_dy : device float max|dY|, or NULL to compute it.
 *   dX      : [M, K], FT_BF16 or FT_F32 (xt).
 *   dA [K, r_l], dB [N, r_l]: float32, overwritten (not accumulated); may be
 *   NULL when r_l == 0.                                                    */
ft_status ft_linear_bwd(const ft_linear* L, const void* dY, const void* X, const void* P_save,
                        int64_t M, const float* amax_dy, void* dX, ft_dtype xt, float* dA,
                        float* dB, void* ws, size_t ws_bytes, void* stream);

/* ft_mlp_fwd -- the forward of a DiT MLP whose two linears are triple-
 * branch layers, with MLP fusion (section 3.3, "MLP Fusion"): FC1's GEMM
 * applies GELU in its epilogue and quantizes its output for FC2 as the
 * tiles leave, so FC2 runs no quantization pass of its own.
 *   Y_up = up's Eq. 2 output (FP32) rounded to bf16; H = GELU(Y_up) rounded
 *   to bf16 (as ft_gelu_bf16); Y = down's Eq. 2 output on H.
 *   up     : [N_up, K] layer; down: [N, N_up] layer (down->K == up->N);
 *            both FT_W4A4G4.
 *   X      : bf16 [M, K] dense;  amax_x: device max|X|, or NULL (computed).
 *   amax_h : device float, required: the tensor amax that fixes the tensor
 *            scale of Q(H).  The fused kernel quantizes H tile by tile,
 *            before all of H exists, so max|H| cannot be measured first: the
 *            caller passes a bound (e.g. the previous step's max|H|).  Values
 *            above it saturate (block scale 448, codes +-6).
 *   H      : bf16 [M, N_up] out: the down layer's input, for its backward;
 *            32-byte aligned (FT_ERR_ALIGN otherwise).
 *   Y      : [M, N] out, FT_BF16 or FT_F32 (yt).
 *   P_up [M, up r_s + r_l], P_down [M, down r_s + r_l]: bf16 out, the
 *            layers' saved down-projections (NULL when the rank is 0).
 *   amax_h_out: NULL, or a device float >= 0 raised to max(*amax_h_out,
 *            max|H|): the exact amax of this call's H, from FC1's
 *            epilogue, to pass as amax_h on the next step (delayed
 *            scaling).  4-byte aligned.
 *   ws     : ft_mlp_workspace_bytes(up, down, M) bytes, zero-filled once.
 *            After the call it holds Q(H) as the down layer's quantized
 *            activation: at byte offset ft_workspace_bytes(M, up->N, up->K,
 *            up->r_s, up->r_l) rounded up to a multiple of 256 lies the down
 *            layer's workspace, laid out as ft_workspace_qact describes for
 *            (M, down->N, down->K, down->r_s, down->r_l).                  */
ft_status ft_mlp_fwd(const ft_linear* up, const ft_linear* down, const void* X, int64_t M, const float* amax_x,
                     const float* amax_h, void* H, void* Y, ft_dtype yt, void* P_up, void* P_down, float* amax_h_out,
                     void* ws, size_t ws_bytes, void* stream);
size_t ft_mlp_workspace_bytes(const ft_linear* up, const ft_linear* down, int64_t M);

/* Workspace sizes (bytes) for the calls above.  Zero-fill a workspace once
 * after allocating it (e.g. cudaMemsetAsync); calls keep their
 * synchronisation words in it and never need it cleared again, whatever
 * earlier calls (finished, failed or of other shapes) left behind.  A
 * workspace holding arbitrary bytes can make a call's device waits run out
 * (reported by ft_device_error as a timeout) instead of computing. */
size_t ft_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r_s, int64_t r_l);
size_t ft_quantize_workspace_bytes(void);

/* ft_workspace_qact -- where the quantized activation of the last
 * ft_linear_fwd / ft_linear_bwd call lies inside its workspace (byte
 * offsets from the workspace start, for the same M, N, K, r_s, r_l).  Once
 * the call's work has finished on its stream, the workspace holds Q(X) after
 * a forward and Q(dY) after a backward, in the layout of an FT_BLK_1x16
 * ft_fp4 view: codes [M, C/2] at *codes_off, scales [M, C/16] at
 * *scales_off, the tensor scale (one float) at *tscale_off, C = K after a
 * forward and N after a backward.  It is the operand of the 4-bit GEMM
 * (section 3.1, Eq. 2 / section 3.2, Eq. 3), the same bytes ft_quantize
 * would produce; a caller may reuse it (e.g. for a quantized weight
 * gradient) until its next call on the workspace.  Pure host arithmetic.
 * FT_ERR_INVALID_ARG for negative sizes or null outputs.                  */
ft_status ft_workspace_qact(int64_t M, int64_t N, int64_t K, int64_t r_s, int64_t r_l,
                            size_t* codes_off, size_t* scales_off, size_t* tscale_off);

/* Reads and clears the device error word of the current device (a host-
 * synchronous copy on `stream`).  *code receives 0 when no kernel reported a
 * failure; otherwise a nonzero code naming the wait that ran out.  Returns
 * FT_ERR_TIMEOUT when *code != 0.                                          */
ft_status ft_device_error(int* code, void* stream);

/* ft_set_cooperative_quantizer -- launch mode of the single-pass quantizer
 * (the kernel that keeps the whole activation in shared memory and finds
 * the tensor amax through a grid-wide barrier, section 3.3's fused down
 * side).  Its barrier needs every CTA of its grid resident at once; the grid
 * never has more CTAs than the device holds at once (one per SM).
 *   on = 0 (the default): a plain launch with programmatic stream
 *     serialization.  Its CTAs take SMs as the previous kernel's CTAs
 *     retire and wait on the device for that kernel's results; all of them
 *     are resident once it ends, unless a kernel of another stream or
 *     process keeps SMs busy meanwhile, or the process may use only part of
 *     the SMs (an MPS share below 100 %, a green context).  If that lasts longer than the
 *     barrier's wait limit (1 s) the call's results are invalid and
 *     ft_device_error() reports the timeout (code 8); nothing hangs.
 *   on = 1: a cooperative launch: the driver starts the grid only when all
 *     of its CTAs fit at once, which is safe next to other streams' kernels
 *     but starts it only after the previous kernel has fully ended (about
 *     3 us later per call on a B200).
 * Process-wide, for calls made after it returns.  Host-only; always FT_OK. */
ft_status ft_set_cooperative_quantizer(int on);

/* ft_set_gemm_mode -- tiling of the 4-bit GEMMs inside ft_linear_fwd,
 * ft_linear_bwd and ft_mlp_fwd (no counterpart in the paper: a choice of
 * how the hardware runs the same sums).
 *   mode = 0 (the default): pairs of CTAs on the two SMs of a TPC share
 *     each 256 x 256 output tile (a thread-block cluster of two; the MMAs
 *     of the pair read half of the weight tile from each SM), whenever the
 *     activation has more than 128 rows; one CTA per 128 x 256 tile
 *     otherwise.
 *   mode = 1: one CTA per 128 x 256 tile always.
 * Both give the same results.  Process-wide, for calls made after it
 * returns.  Host-only; FT_ERR_INVALID_ARG for another mode. */
ft_status ft_set_gemm_mode(int mode);

/* Human-readable name of a status. */
const char* ft_status_str(ft_status s);

/* ft_linear_fwd_noalloc -- the forward of ft_linear_fwd for callers that
 * cannot allocate device memory or hand over a workspace (a C host with no
 * device allocator, a plug-in inside a framework that owns all device memory
 * through its own pool, code that must not allocate while queueing work).
 * The paper has no counterpart: this is a deployment convenience.
 *   Arguments, results and errors are those of ft_linear_fwd, without ws.
 *   Scratch: a fixed array inside the library's device image,
 *   ft_linear_fwd_noalloc_max_bytes() = 32 MiB, held on every GPU that
 *   loads the library until the process exits.  A layer/batch whose
 *   ft_workspace_bytes() exceeds it returns FT_ERR_WORKSPACE, nothing
 *   launched.  The function itself allocates nothing.
 *   The first call on a device looks up the array's device address (once
 *   per device, with that device current, and again in a new context of the
 *   device after cudaDeviceReset); make that first call before any stream
 *   capture.
 *   All calls on a device share its one copy of the array, which keeps the
 *   last call's contents (each call clears what must start at zero itself).
 *   Calls whose work overlaps on the same GPU (two streams, two host
 *   threads) race on the array: the caller must serialise them.  Calls on
 *   different GPUs use different copies.                                  */
ft_status ft_linear_fwd_noalloc(const ft_linear* L, const void* X, int64_t M, const float* amax_x,
                                void* Y, ft_dtype yt, void* P_save, void* stream);
size_t ft_linear_fwd_noalloc_max_bytes(void);

/* Measurement support (no counterpart in the method; used to report each
 * kernel's roofline fraction from inside a real step).  While enabled, every
 * kernel launch of the library is bracketed by two CUDA events on its
 * stream.  ft_timing_read() waits for the recorded events, adds their
 * elapsed times to per-kernel totals and returns the total milliseconds and
 * launch count of one kernel (by name, e.g. "k_gemm_fp4"; "*" = all
 * kernels).  ft_timing_reset() clears the totals.  Host-synchronous; not
 * for use inside stream capture.                                          */
ft_status ft_timing_enable(int on);
ft_status ft_timing_read(const char* kernel, double* total_ms, int64_t* launches);
ft_status ft_timing_reset(void);

#ifdef __cplusplus
}
#endif
#endif /* FT_H_ */
