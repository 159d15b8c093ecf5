"""B200-native W4A4G4 triple-branch linear layer (FourTune).

Thin Python binding over the C ABI of include/ft.h.  Every function here only
marshals torch CUDA tensors into pointers and calls the CUDA library; all
arithmetic of the hot path runs in the library's sm_100a kernels.  PyTorch is
used for device memory and streams.

    layer = prepare_layer(W, r_s=32, A=A, B=B, s=1.0)    # once per layer
    Y, P  = ft_linear_fwd(layer, X)                       # Eq. 2
    dX, dA, dB = ft_linear_bwd(layer, dY, X, P)           # Eq. 3 + adapter grads
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from ._lib import FtFp4, FtLinear, FtError, check, load

BLK_1x16 = 0
BLK_16x16 = 1
BF16 = 0
F32 = 1
# precision configurations (the FourTune page's Table 4); the weight is
# always 4-bit, bit 0 = 16-bit activations, bit 1 = 16-bit gradients
W4A4G4, W4A16G4, W4A4G16, W4A16G16 = 0, 1, 2, 3
PRECISIONS = {"W4A4G4": W4A4G4, "W4A16G4": W4A16G4, "W4A4G16": W4A4G16, "W4A16G16": W4A16G16}

__all__ = [
    "FP4", "Layer", "FtError", "BLK_1x16", "BLK_16x16", "BF16", "F32",
    "W4A4G4", "W4A16G4", "W4A4G16", "W4A16G16", "PRECISIONS", "ft_dequant_weight_operands", "ft_gelu_bf16",
    "ft_mlp_fwd", "ft_mlp_workspace_bytes",
    "ft_quantize", "ft_quantize_transpose", "ft_linear_fwd", "ft_linear_bwd",
    "ft_workspace_bytes", "ft_quantize_workspace_bytes", "ft_device_error",
    "ft_set_cooperative_quantizer", "ft_set_gemm_mode", "GEMM_PAIRS", "GEMM_SINGLE", "prepare_layer", "svd_split", "Workspace", "timing",
]


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
    return t


@dataclass
class FP4:
    """NVFP4 tensor: codes [rows, cols/2] uint8, scales (E4M3 bytes) and the
    decode tensor scale (1 float), all device tensors."""
    codes: torch.Tensor
    scales: torch.Tensor
    tscale: torch.Tensor
    rows: int
    cols: int
    blk: int

    @staticmethod
    def empty(rows: int, cols: int, blk: int, device, scales=None, tscale=None) -> "FP4":
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=device)
        if scales is None:
            sshape = (rows, cols // 16) if blk == BLK_1x16 else (rows // 16, cols // 16)
            scales = torch.empty(sshape, dtype=torch.uint8, device=device)
        if tscale is None:
            tscale = torch.empty(1, dtype=torch.float32, device=device)
        return FP4(codes, scales, tscale, rows, cols, blk)

    def view(self) -> FtFp4:
        return FtFp4(self.codes.data_ptr(), _ptr(self.scales), _ptr(self.tscale), self.rows,
                     self.cols, self.blk)


class Workspace:
    """Caller-owned scratch for the library (it never allocates)."""

    def __init__(self):
        self.buf = None

    def get(self, nbytes: int, device) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != torch.device(device):
            # zero-filled once: the library's synchronisation words live here
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self.buf


_default_ws: dict = {}


def _ws(ws, nbytes, device):
    if ws is None:
        key = torch.device(device)
        ws = _default_ws.setdefault(key, Workspace())
    return ws.get(nbytes, device)


def ft_workspace_bytes(M: int, N: int, K: int, r_s: int, r_l: int) -> int:
    return load().ft_workspace_bytes(M, N, K, r_s, r_l)


def ft_quantize_workspace_bytes() -> int:
    return load().ft_quantize_workspace_bytes()


def ft_workspace_qact(M: int, N: int, K: int, r_s: int, r_l: int) -> tuple[int, int, int]:
    """Byte offsets (codes, scales, tensor scale) of the quantized
    activation that ft_linear_fwd (Q(X)) or ft_linear_bwd (Q(dY)) leaves in
    its workspace."""
    c, s, g = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    check("ft_workspace_qact", load().ft_workspace_qact(M, N, K, r_s, r_l, ctypes.byref(c),
                                                        ctypes.byref(s), ctypes.byref(g)))
    return c.value, s.value, g.value


def ft_quantize(x: torch.Tensor, blk: int = BLK_1x16, amax: torch.Tensor | None = None,
                out: FP4 | None = None, ws: Workspace | None = None, stream=None) -> FP4:
    """Q(x): NVFP4 block quantization of a 2-D bf16 CUDA tensor."""
    _bf16(x, "x")
    rows, cols = x.shape
    if x.stride(1) != 1:
        raise ValueError("x must have unit column stride")
    out = out or FP4.empty(rows, cols, blk, x.device)
    wbuf = _ws(ws, ft_quantize_workspace_bytes(), x.device) if amax is None else None
    v = out.view()
    check("ft_quantize", load().ft_quantize(
        x.data_ptr(), rows, cols, x.stride(0), blk, _ptr(amax), ctypes.byref(v), _ptr(wbuf),
        0 if wbuf is None else wbuf.numel(), _stream(stream)))
    return out


def ft_quantize_transpose(x: torch.Tensor, blk: int = BLK_16x16, amax: torch.Tensor | None = None,
                          out_row: FP4 | None = None, out_col: FP4 | None = None,
                          ws: Workspace | None = None, stream=None):
    """Both layouts in one pass.  16x16: (codes packed along rows, the same
    codes transposed) sharing one scale grid.  1x16: (Q(x), Q(x^T))."""
    _bf16(x, "x")
    rows, cols = x.shape
    out_row = out_row or FP4.empty(rows, cols, blk, x.device)
    if out_col is None:
        if blk == BLK_16x16:
            out_col = FP4.empty(cols, rows, blk, x.device, scales=out_row.scales, tscale=out_row.tscale)
        else:
            out_col = FP4.empty(cols, rows, blk, x.device)
    wbuf = _ws(ws, ft_quantize_workspace_bytes(), x.device) if amax is None else None
    vr, vc = out_row.view(), out_col.view()
    check("ft_quantize_transpose", load().ft_quantize_transpose(
        x.data_ptr(), rows, cols, x.stride(0), blk, _ptr(amax), ctypes.byref(vr), ctypes.byref(vc),
        _ptr(wbuf), 0 if wbuf is None else wbuf.numel(), _stream(stream)))
    return out_row, out_col


@dataclass
class Layer:
    """One triple-branch linear: Q(W_res) in both code layouts (one scale
    grid), the stabilizer factors U [K, r_s], V [N, r_s] and the adapter
    A [K, r_l], B [N, r_l] (bf16), and the LoRA scale s."""
    N: int
    K: int
    r_s: int
    r_l: int
    s: float
    w_k: FP4
    w_n: FP4
    U: torch.Tensor | None
    V: torch.Tensor | None
    A: torch.Tensor | None
    B: torch.Tensor | None
    op_k: torch.Tensor | None = None  # the GEMM's image of w_k (codes + per-row scales)
    op_n: torch.Tensor | None = None  # ... and of w_n
    precision: int = W4A4G4           # W4A4G4 (the method) or a 16-bit variant
    wd_k: torch.Tensor | None = None  # bf16 image of Q(W_res) [N, K] (16-bit activations)
    wd_n: torch.Tensor | None = None  # ... transposed [K, N] (16-bit gradients)

    def view(self) -> FtLinear:
        return FtLinear(self.N, self.K, self.r_s, self.r_l, self.s, self.w_k.view(), self.w_n.view(),
                        _ptr(self.U), _ptr(self.V), _ptr(self.A), _ptr(self.B), _ptr(self.op_k),
                        _ptr(self.op_n), int(self.precision), _ptr(self.wd_k), _ptr(self.wd_n))


def _bf16_rne(x: torch.Tensor) -> torch.Tensor:
    """float64 -> bf16 with one round-to-nearest-even step (torch's own cast
    goes through float32 and so rounds twice, which differs at near-ties):
    the value is scaled so that bf16's 8 significant bits are the integer
    part, rounded half to even, and scaled back -- exact in bf16 from there."""
    _, e = torch.frexp(x)
    q = torch.clamp(e.to(torch.int64) - 8, min=-133)
    return torch.ldexp(torch.round(torch.ldexp(x, -q)), q).to(torch.float32).to(torch.bfloat16)


def svd_split(W: torch.Tensor, r_s: int):
    """Eq. 1 on the host side (untimed, once per layer): W ~ W_res + V U^T
    with the top-r_s singular triplets, taken from the smaller Gram matrix in
    float64 (eigenvectors of W^T W are the right singular vectors, those of
    W W^T the left ones).  U = right vectors [K, r_s], V = W U [N, r_s], both
    rounded to bf16, and W_res = W - V U^T from the rounded factors (each
    rounded once, to nearest even)."""
    Wd = W.to(torch.float64)
    N, K = Wd.shape
    if r_s == 0:
        return None, None, W.to(torch.bfloat16).contiguous()
    if K <= N:
        evals, evecs = torch.linalg.eigh(Wd.T @ Wd)
        vtop = evecs[:, torch.argsort(evals, descending=True)[:r_s]]
    else:
        evals, evecs = torch.linalg.eigh(Wd @ Wd.T)
        order = torch.argsort(evals, descending=True)[:r_s]
        sig = evals[order].clamp_min(0).sqrt()
        vtop = (Wd.T @ evecs[:, order]) / torch.where(sig > 0, sig, torch.ones_like(sig))
    U = _bf16_rne(vtop).contiguous()
    V = _bf16_rne(Wd @ U.to(torch.float64)).contiguous()
    W_res = _bf16_rne(Wd - V.to(torch.float64) @ U.to(torch.float64).T).contiguous()
    return U, V, W_res


def prepare_layer(W: torch.Tensor | None = None, r_s: int = 0, A: torch.Tensor | None = None,
                  B: torch.Tensor | None = None, s: float = 1.0, *, U=None, V=None, W_res=None,
                  amax: torch.Tensor | None = None, ws: Workspace | None = None,
                  weight_blk: int = BLK_16x16, precision: int | str = W4A4G4) -> Layer:
    """Once-per-layer preparation: split W (or take a given U, V, W_res) and
    quantize W_res into both code layouts in one pass: 16x16 blocks (the
    method), or with weight_blk=BLK_1x16 the granularity ablation's 1x16
    groups (W_res along K and, independently, W_res^T along N).  precision:
    W4A4G4 (the method) or a 16-bit variant ("W4A16G4", "W4A4G16",
    "W4A16G16"), for which the bf16 weight images are built as well."""
    if W_res is None:
        U, V, W_res = svd_split(W, r_s)
    _bf16(W_res, "W_res")
    N, K = W_res.shape
    r_s = 0 if U is None else U.shape[1]
    r_l = 0 if A is None else A.shape[1]
    w_k, w_n = ft_quantize_transpose(W_res.contiguous(), weight_blk, amax=amax, ws=ws)
    op_k, op_n = ft_pack_weight_operands(w_k, w_n, N, K)
    prec = PRECISIONS[precision] if isinstance(precision, str) else int(precision)
    wd_k, wd_n = ft_dequant_weight_operands(w_k, w_n, fwd=bool(prec & W4A16G4), dgrad=bool(prec & W4A4G16))
    return Layer(N, K, r_s, r_l, float(s), w_k, w_n, U, V,
                 None if A is None else A.contiguous(), None if B is None else B.contiguous(), op_k, op_n,
                 prec, wd_k, wd_n)


def ft_dequant_weight_operands(w_k: FP4, w_n: FP4, fwd: bool = True, dgrad: bool = True, stream=None):
    """bf16 images of Q(W_res) for the 16-bit GEMMs of the precision
    variants: (wd_k [N, K] if fwd, wd_n [K, N] if dgrad), e2m1 value x block
    scale (exact; the tensor scale stays in w_k.tscale).  (None, None) when
    neither is asked for."""
    if not fwd and not dgrad:
        return None, None
    dev = w_k.codes.device
    wd_k = torch.empty(w_k.rows, w_k.cols, dtype=torch.bfloat16, device=dev) if fwd else None
    wd_n = torch.empty(w_k.cols, w_k.rows, dtype=torch.bfloat16, device=dev) if dgrad else None
    vk, vn = w_k.view(), w_n.view()
    check("ft_dequant_weight_operands", load().ft_dequant_weight_operands(
        ctypes.byref(vk), ctypes.byref(vn), _ptr(wd_k), _ptr(wd_n), _stream(stream)))
    return wd_k, wd_n


def ft_pack_weight_operands(w_k, w_n, N: int, K: int, stream=None):
    """The 4-bit GEMMs' images of Q(W_res) in both orientations: codes and the
    16x16 scales repeated per row, side by side per 256 x 256 block.  Returns
    (op_k, op_n), uint8."""
    nbytes = load().ft_weight_operand_bytes(N, K)
    op_k = torch.empty(nbytes, dtype=torch.uint8, device=w_k.codes.device)
    op_n = torch.empty(nbytes, dtype=torch.uint8, device=w_k.codes.device)
    if w_k.blk == BLK_1x16:
        check("ft_pack_weight_operands_1x16", load().ft_pack_weight_operands_1x16(
            w_k.codes.data_ptr(), w_k.scales.data_ptr(), w_n.codes.data_ptr(), w_n.scales.data_ptr(), N, K,
            op_k.data_ptr(), op_n.data_ptr(), _stream(stream)))
    else:
        check("ft_pack_weight_operands", load().ft_pack_weight_operands(
            w_k.codes.data_ptr(), w_n.codes.data_ptr(), w_k.scales.data_ptr(), N, K, op_k.data_ptr(),
            op_n.data_ptr(), _stream(stream)))
    return op_k, op_n


def ft_linear_fwd(layer: Layer, X: torch.Tensor, amax_x: torch.Tensor | None = None,
                  out_dtype: int = BF16, Y: torch.Tensor | None = None, P: torch.Tensor | None = None,
                  ws: Workspace | None = None, stream=None, amax_y: torch.Tensor | None = None):
    """Y = Q(X) Q(W_res)^T + (X U) V^T + s (X A) B^T.  Returns (Y, P) where
    P = [bf16(X U) | bf16(s X A)] is saved for the backward.  amax_y: an
    optional float32 device scalar (>= 0) raised to max|Y| by the GEMM's
    epilogue."""
    _bf16(X, "X")
    M = X.shape[0]
    r = layer.r_s + layer.r_l
    if Y is None:
        Y = torch.empty(M, layer.N, device=X.device,
                        dtype=torch.float32 if out_dtype == F32 else torch.bfloat16)
    if P is None:
        P = torch.empty(M, max(r, 0), device=X.device, dtype=torch.bfloat16)
    wbuf = _ws(ws, ft_workspace_bytes(M, layer.N, layer.K, layer.r_s, layer.r_l), X.device)
    v = layer.view()
    check("ft_linear_fwd", load().ft_linear_fwd(
        ctypes.byref(v), X.data_ptr(), M, _ptr(amax_x), Y.data_ptr(), out_dtype,
        P.data_ptr() if r > 0 else None, _ptr(amax_y), wbuf.data_ptr(), wbuf.numel(), _stream(stream)))
    return Y, P


def ft_linear_bwd(layer: Layer, dY: torch.Tensor, X: torch.Tensor, P: torch.Tensor,
                  amax_dy: torch.Tensor | None = None, out_dtype: int = BF16,
                  dX: torch.Tensor | None = None, dA: torch.Tensor | None = None,
                  dB: torch.Tensor | None = None, ws: Workspace | None = None, stream=None):
    """dX = Q(dY) Q(W_res) + (dY V) U^T + s (dY B) A^T;  dB = dY^T P_lora,
    dA = X^T Pg_lora (float32, overwritten).  Returns (dX, dA, dB)."""
    _bf16(dY, "dY")
    M = dY.shape[0]
    r = layer.r_s + layer.r_l
    if dX is None:
        dX = torch.empty(M, layer.K, device=dY.device,
                         dtype=torch.float32 if out_dtype == F32 else torch.bfloat16)
    if layer.r_l > 0:
        dA = dA if dA is not None else torch.empty(layer.K, layer.r_l, device=dY.device, dtype=torch.float32)
        dB = dB if dB is not None else torch.empty(layer.N, layer.r_l, device=dY.device, dtype=torch.float32)
    wbuf = _ws(ws, ft_workspace_bytes(M, layer.N, layer.K, layer.r_s, layer.r_l), dY.device)
    v = layer.view()
    check("ft_linear_bwd", load().ft_linear_bwd(
        ctypes.byref(v), dY.data_ptr(), _ptr(X), P.data_ptr() if r > 0 else None, M, _ptr(amax_dy),
        dX.data_ptr(), out_dtype, _ptr(dA), _ptr(dB), wbuf.data_ptr(), wbuf.numel(), _stream(stream)))
    return dX, dA, dB


def ft_mlp_workspace_bytes(up: Layer, down: Layer, M: int) -> int:
    vu, vd = up.view(), down.view()
    return load().ft_mlp_workspace_bytes(ctypes.byref(vu), ctypes.byref(vd), M)


def ft_mlp_fwd(up: Layer, down: Layer, X: torch.Tensor, amax_h: torch.Tensor, amax_x: torch.Tensor | None = None,
               out_dtype: int = BF16, H: torch.Tensor | None = None, Y: torch.Tensor | None = None,
               P_up: torch.Tensor | None = None, P_down: torch.Tensor | None = None,
               ws: Workspace | None = None, stream=None, amax_h_out: torch.Tensor | None = None):
    """The MLP forward with FC1's GEMM fused with FC2's quantization: H =
    GELU(bf16(FC1(X))) and Y = FC2(H), Q(H) made by FC1's epilogue with the
    tensor scale of the supplied amax_h.  amax_h_out: an optional float32
    device scalar (>= 0) raised to max|H| (the next step's amax_h).
    Returns (Y, H, P_up, P_down)."""
    _bf16(X, "X")
    M = X.shape[0]
    dev = X.device
    H = torch.empty(M, up.N, dtype=torch.bfloat16, device=dev) if H is None else H
    if Y is None:
        Y = torch.empty(M, down.N, device=dev, dtype=torch.float32 if out_dtype == F32 else torch.bfloat16)
    ru, rd = up.r_s + up.r_l, down.r_s + down.r_l
    P_up = torch.empty(M, max(ru, 0), dtype=torch.bfloat16, device=dev) if P_up is None else P_up
    P_down = torch.empty(M, max(rd, 0), dtype=torch.bfloat16, device=dev) if P_down is None else P_down
    wbuf = _ws(ws, ft_mlp_workspace_bytes(up, down, M), dev)
    vu, vd = up.view(), down.view()
    check("ft_mlp_fwd", load().ft_mlp_fwd(
        ctypes.byref(vu), ctypes.byref(vd), X.data_ptr(), M, _ptr(amax_x), amax_h.data_ptr(), H.data_ptr(),
        Y.data_ptr(), out_dtype, P_up.data_ptr() if ru > 0 else None, P_down.data_ptr() if rd > 0 else None,
        _ptr(amax_h_out), wbuf.data_ptr(), wbuf.numel(), _stream(stream)))
    return Y, H, P_up, P_down


def ft_gelu_bf16(y: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """h = GELU(y) on bf16, each value correctly rounded (the activation the
    fused MLP applies between its linears)."""
    _bf16(y, "y")
    if not y.is_contiguous():
        raise ValueError("y must be contiguous")
    out = torch.empty_like(y) if out is None else out
    check("ft_gelu_bf16", load().ft_gelu_bf16(y.data_ptr(), out.data_ptr(), y.numel(), _stream(stream)))
    return out


def ft_device_error(stream=None) -> int:
    """Reads and clears the device error word (0 = no kernel reported a
    bounded wait that ran out)."""
    code = ctypes.c_int(0)
    load().ft_device_error(ctypes.byref(code), _stream(stream))
    return code.value


def ft_set_cooperative_quantizer(on: bool) -> None:
    """Launch mode of the single-pass quantizer's grid barrier: False (the
    default) = plain launch, True = cooperative launch (safe next to other
    streams' long-running kernels, ~3 us later start per call)."""
    check("ft_set_cooperative_quantizer", load().ft_set_cooperative_quantizer(1 if on else 0))


GEMM_PAIRS, GEMM_SINGLE = 0, 1


def ft_set_gemm_mode(mode: int) -> None:
    """Tiling of the 4-bit GEMMs: GEMM_PAIRS (the default: CTA pairs share
    256 x 256 tiles when the activation has more than 128 rows) or
    GEMM_SINGLE (one CTA per 128 x 256 tile).  Same results either way."""
    check("ft_set_gemm_mode", load().ft_set_gemm_mode(int(mode)))


class timing:
    """Per-kernel CUDA-event timing of the library's launches (measurement)."""

    @staticmethod
    def enable(on: bool = True) -> None:
        check("ft_timing_enable", load().ft_timing_enable(1 if on else 0))

    @staticmethod
    def reset() -> None:
        check("ft_timing_reset", load().ft_timing_reset())

    @staticmethod
    def read(kernel: str = "*"):
        """(total milliseconds, launches) of one kernel since the last reset."""
        ms = ctypes.c_double(0.0)
        n = ctypes.c_int64(0)
        check("ft_timing_read", load().ft_timing_read(kernel.encode(), ctypes.byref(ms), ctypes.byref(n)))
        return ms.value, n.value
