"""CPU oracle for the FourTune W4A4G4 triple-branch linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  The
CUDA library never loads it and shares no code with it.

Sources (page "FourTune: Towards Fully 4-Bit Efficient Post-Training for
Diffusion Models"):
  * Eq. 1 (section 3.1): W ~ R + L_stab with L_stab = L1 L2 from the SVD.
  * Eq. 2 (section 3.1): Y = GEMM4(Q(X), Q(R)) + X L_stab + X (A B).
  * Eq. 3 (section 3.2): dX = GEMM4(Q(G), Q(R)^T) + G L_stab^T + G (A B)^T.
  * Section 3.2, LoRA gradients: dB = (X A)^T G, dA = X^T (G B^T).
  * Section 3.2: 16x16 weight blocks, so Q(R)^T is the transposed codes with
    the same scales.

Convention (PyTorch style, weights stored [out, in]):
  W, W_res: [N, K];  U: [K, r_s];  V: [N, r_s];  A: [K, r_l];  B: [N, r_l]
  Y = Q(X) Q(W_res)^T + (X U) V^T + s (X A) B^T
so L_stab = (U V^T)^T in the page's notation and the page's R is W_res^T.

The bit-level quantizer lives in ``ft_oracle.c`` (plain C, compiled with
gcc -O2 -ffp-contract=off, no fast-math).  The contractions here use numpy's
float64 matmul as a library primitive on the dequantized operands; nothing
is blocked, fused or reordered beyond the equations above.

Rounding points (the page is silent; plainest reading):
  P   = [bf16(X U) | bf16(s * (X A))]          saved for the backward
  Pg  = [bf16(dY V) | bf16(s * (dY B))]
  Y, dX in float64;  dA = X^T Pg_lora,  dB = dY^T P_lora in float64.
The low-rank branches read the unquantized bf16 X and dY (Eq. 2 and Eq. 3
apply Q only inside GEMM4).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ft_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libft_oracle.so")

_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile ft_oracle.c into a shared library (gcc, IEEE single, no FMA)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.fto_e2m1_value.restype = ctypes.c_double
        L.fto_e2m1_value.argtypes = [ctypes.c_uint8]
        L.fto_e2m1_encode.restype = ctypes.c_uint8
        L.fto_e2m1_encode.argtypes = [ctypes.c_float]
        L.fto_e4m3_value.restype = ctypes.c_double
        L.fto_e4m3_value.argtypes = [ctypes.c_uint8]
        L.fto_e4m3_encode.restype = ctypes.c_uint8
        L.fto_e4m3_encode.argtypes = [ctypes.c_float]
        L.fto_amax_bf16.restype = ctypes.c_float
        L.fto_amax_bf16.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.fto_tensor_scale.restype = ctypes.c_float
        L.fto_tensor_scale.argtypes = [ctypes.c_float]
        L.fto_quantize_1x16.restype = None
        L.fto_quantize_1x16.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_float, _u8p, _u8p,
                                        ctypes.POINTER(ctypes.c_float)]
        L.fto_quantize_16x16.restype = None
        L.fto_quantize_16x16.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_float, _u8p, ctypes.c_void_p, _u8p,
                                         ctypes.POINTER(ctypes.c_float)]
        L.fto_dequant_1x16.restype = None
        L.fto_dequant_1x16.argtypes = [_u8p, _u8p, ctypes.c_float, ctypes.c_int64,
                                       ctypes.c_int64, _f64p]
        L.fto_dequant_16x16.restype = None
        L.fto_dequant_16x16.argtypes = [_u8p, _u8p, ctypes.c_float, ctypes.c_int64,
                                        ctypes.c_int64, _f64p]
        L.fto_gemm_nt_f64.restype = None
        L.fto_gemm_nt_f64.argtypes = [_f64p, _f64p, ctypes.c_int64, ctypes.c_int64, _i64p,
                                      ctypes.c_int64, _f64p]
        _lib = L
    return _lib


# ------------------------------------------------------------------ formats

def e2m1_value(code: int) -> float:
    return lib().fto_e2m1_value(code)


def e2m1_encode(q: float) -> int:
    return lib().fto_e2m1_encode(q)


def e4m3_value(byte: int) -> float:
    return lib().fto_e4m3_value(byte)


def e4m3_encode(v: float) -> int:
    return lib().fto_e4m3_encode(v)


# --------------------------------------------------------------------- bf16

def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns."""
    u32 = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


def bf16_from_f64(v) -> np.ndarray:
    """Round float64 values to bf16 (round-to-nearest-even), as bit patterns.

    bf16 keeps 8 significant bits; the rounding quantum of a value with
    binary exponent e (v = m 2^e, 0.5 <= |m| < 1) is 2^(e-8), and never finer
    than the subnormal quantum 2^-133.  Scaling by powers of two is exact, so
    np.rint performs exactly one RNE rounding.
    """
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    q = np.maximum(e - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(v, -q)), q)
    with np.errstate(over="ignore"):
        f = r.astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


# ------------------------------------------------------------- quantization

def amax_bf16(x: np.ndarray) -> float:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    return float(lib().fto_amax_bf16(x, x.shape[0], x.shape[1], x.shape[1]))


def tensor_scale(amax: float) -> float:
    return float(lib().fto_tensor_scale(amax))


def quantize_1x16(x: np.ndarray, amax: float | None = None):
    """1x16 NVFP4 quantization along rows.  Returns (codes, scales, g)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = x.shape
    assert cols % 16 == 0
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    g = ctypes.c_float(0.0)
    lib().fto_quantize_1x16(x, rows, cols, cols, -1.0 if amax is None else float(amax),
                            codes, scales, ctypes.byref(g))
    return codes, scales, float(np.float32(g.value))


def quantize_16x16(x: np.ndarray, amax: float | None = None, want_col: bool = True):
    """16x16 NVFP4 quantization.  Returns (codes_row, codes_col, scales, g);
    codes_col holds the same codes packed along columns (the transpose)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = x.shape
    assert rows % 16 == 0 and cols % 16 == 0
    codes_row = np.zeros((rows, cols // 2), np.uint8)
    codes_col = np.zeros((cols, rows // 2), np.uint8) if want_col else None
    scales = np.zeros((rows // 16, cols // 16), np.uint8)
    g = ctypes.c_float(0.0)
    col_ptr = codes_col.ctypes.data_as(ctypes.c_void_p) if want_col else None
    lib().fto_quantize_16x16(x, rows, cols, cols, -1.0 if amax is None else float(amax),
                             codes_row, col_ptr, scales, ctypes.byref(g))
    return codes_row, codes_col, scales, float(np.float32(g.value))


def quantize_1x16_colwise(x: np.ndarray, amax: float | None = None):
    """Column-wise copy: 1x16 quantization of x^T (blocks run along the rows
    of x), sharing the tensor scale of x."""
    if amax is None:
        amax = amax_bf16(x)
    return quantize_1x16(np.ascontiguousarray(np.asarray(x).T), amax)


def dequant_1x16(codes, scales, g, rows, cols) -> np.ndarray:
    out = np.empty((rows, cols), np.float64)
    lib().fto_dequant_1x16(np.ascontiguousarray(codes), np.ascontiguousarray(scales),
                           float(g), rows, cols, out)
    return out


def dequant_16x16(codes_row, scales, g, rows, cols) -> np.ndarray:
    out = np.empty((rows, cols), np.float64)
    lib().fto_dequant_16x16(np.ascontiguousarray(codes_row), np.ascontiguousarray(scales),
                            float(g), rows, cols, out)
    return out


def gemm_nt_plain(A: np.ndarray, B: np.ndarray, rows=None) -> np.ndarray:
    """C = A[rows] B^T by a plain triple loop in C (FP64)."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    idx = np.arange(A.shape[0], dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    C = np.empty((len(idx), B.shape[0]), np.float64)
    lib().fto_gemm_nt_f64(A, B, A.shape[1], B.shape[0], np.ascontiguousarray(idx), len(idx), C)
    return C


# -------------------------------------------------------------- weight prep

def svd_split(W: np.ndarray, r_s: int):
    """Eq. 1: W ~ W_res + V U^T with the top-r_s singular triplets.

    The top singular subspace comes from the smaller Gram matrix: with
    W = sum_i sigma_i u_i v_i^T, the eigenvectors of W^T W are the v_i and
    those of W W^T the u_i (eigenvalues sigma_i^2).  U = [v_i] [K, r_s] and
    V = [sigma_i u_i] = W U [N, r_s].  U and V are rounded to bf16 first and
    W_res = W - V U^T is formed from the rounded factors, so W_res + V U^T
    reproduces W up to the bf16 rounding of W_res.  Returns bf16 bit patterns
    (U, V, W_res).
    """
    Wd = bf16_to_f64(W)
    N, K = Wd.shape
    if r_s == 0:
        return (np.zeros((K, 0), np.uint16), np.zeros((N, 0), np.uint16), np.asarray(W, np.uint16))
    if K <= N:
        evals, evecs = np.linalg.eigh(Wd.T @ Wd)
        vtop = evecs[:, np.argsort(evals)[::-1][:r_s]]
    else:
        evals, evecs = np.linalg.eigh(Wd @ Wd.T)
        order = np.argsort(evals)[::-1][:r_s]
        utop = evecs[:, order]
        sig = np.sqrt(np.maximum(evals[order], 0.0))
        vtop = (Wd.T @ utop) / np.where(sig > 0, sig, 1.0)
    U = bf16_from_f64(vtop)
    V = bf16_from_f64(Wd @ bf16_to_f64(U))
    W_res = bf16_from_f64(Wd - bf16_to_f64(V) @ bf16_to_f64(U).T)
    return U, V, W_res


# -------------------------------------------------------------- layer math

def _lowrank_down(Xd: np.ndarray, L1: np.ndarray, L2: np.ndarray, s: float):
    """[bf16(X L1) | bf16(s (X L2))] from float64 values (bf16 inputs)."""
    parts = []
    if L1.shape[1]:
        parts.append(bf16_from_f64(Xd @ bf16_to_f64(L1)))
    if L2.shape[1]:
        parts.append(bf16_from_f64(s * (Xd @ bf16_to_f64(L2))))
    if not parts:
        return np.zeros((Xd.shape[0], 0), np.uint16)
    return np.concatenate(parts, axis=1)


def _weight_fwd(W_res, qw, weight_blk):
    """Dequantized forward weight [N, K]: 16x16 blocks (the method's), or
    1x16 groups along K (the granularity ablation: FourTune page, section 4,
    "Impact of Quantization Granularity", Table 5)."""
    N, K = W_res.shape
    if weight_blk == "16x16":
        qw = quantize_16x16(W_res) if qw is None else qw
        return qw, dequant_16x16(qw[0], qw[2], qw[3], N, K)
    if weight_blk == "1x16":
        qw = quantize_1x16(W_res) if qw is None else qw
        return qw, dequant_1x16(qw[0], qw[1], qw[2], N, K)
    raise ValueError(weight_blk)


def _weight_dgrad(W_res, qw, weight_blk):
    """Dequantized dgrad weight as [N, K]: the 16x16 codes serve both
    directions (their blocks are square); 1x16 groups along K do not, so
    W_res^T is quantized again in 1x16 groups along N (same tensor scale)."""
    N, K = W_res.shape
    if weight_blk == "16x16":
        qw = quantize_16x16(W_res) if qw is None else qw
        return qw, dequant_16x16(qw[0], qw[2], qw[3], N, K)
    if weight_blk == "1x16":
        qw = quantize_1x16_colwise(W_res) if qw is None else qw
        return qw, dequant_1x16(qw[0], qw[1], qw[2], K, N).T
    raise ValueError(weight_blk)


PRECISIONS = ("W4A4G4", "W4A16G4", "W4A4G16", "W4A16G16")


def _act_bits(precision: str) -> int:
    """Bits of the activations in the forward GEMM (FourTune page, section
    4, "Impact of Precision Configurations", Table 4: W4A4G4 is the method;
    W4A16G4, W4A4G16 and W4A16G16 keep activations and/or gradients at 16
    bits, the weight always 4-bit)."""
    if precision not in PRECISIONS:
        raise ValueError(precision)
    return 16 if "A16" in precision else 4


def _grad_bits(precision: str) -> int:
    """Bits of the output gradients in the dgrad GEMM (Table 4, as above)."""
    if precision not in PRECISIONS:
        raise ValueError(precision)
    return 16 if "G16" in precision else 4


def linear_fwd(X, W_res, U, V, A, B, s: float, rows=None, amax_x=None, qw=None, weight_blk="16x16",
               precision="W4A4G4"):
    """Forward of the triple-branch layer (Eq. 2).

    X: bf16 [M, K]; W_res: bf16 [N, K]; U [K, r_s]; V [N, r_s]; A [K, r_l];
    B [N, r_l].  rows: optional row sample for Y (the quantization and P are
    always computed on the full tensors).  weight_blk: "16x16" (the method)
    or "1x16" (groups along K, the granularity ablation).  qw: optional
    precomputed quantize_16x16(W_res) (resp. quantize_1x16(W_res)).
    precision: one of PRECISIONS; with 16-bit activations (W4A16G*) the
    backbone GEMM reads X itself instead of Q(X) (qx is then None).
    Returns a dict with Y (float64 [len(rows), N]), P (bf16 [M, r_s + r_l]),
    qx = (codes, scales, g) and qw.
    """
    M, K = X.shape
    N = W_res.shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    qw, Wq = _weight_fwd(W_res, qw, weight_blk)
    Xd = bf16_to_f64(X)
    if _act_bits(precision) == 16:
        qx = None
        Xq = Xd[rows]
    else:
        qx = quantize_1x16(X, amax_x)
        Xq = dequant_1x16(qx[0], qx[1], qx[2], M, K)[rows]
    P = _lowrank_down(Xd, U, A, s)
    Pd = bf16_to_f64(P[rows])
    LR = np.concatenate([bf16_to_f64(V), bf16_to_f64(B)], axis=1)  # [N, r_s + r_l]
    Y = Xq @ Wq.T + Pd @ LR.T
    return {"Y": Y, "P": P, "qx": qx, "qw": qw, "rows": rows}


def linear_bwd(dY, X, W_res, U, V, A, B, s: float, P, rows=None, amax_dy=None, qw=None,
               weight_blk="16x16", precision="W4A4G4"):
    """Backward of the triple-branch layer (Eq. 3 and the LoRA gradients).

    dY: bf16 [M, N]; X: bf16 [M, K]; P: the forward's saved bf16 [M, r_s+r_l].
    weight_blk as in linear_fwd; qw: optional precomputed quantize_16x16(W_res)
    (resp. quantize_1x16_colwise(W_res), the dgrad operand of 1x16 weights).
    precision: one of PRECISIONS; with 16-bit gradients (W4A*G16) the dgrad
    GEMM reads dY itself instead of Q(dY) (qdy is then None).
    Returns dX (float64 [len(rows), K]), dA (float64 [K, r_l]),
    dB (float64 [N, r_l]), Pg (bf16 [M, r_s + r_l]) and qdy.
    """
    M, N = dY.shape
    K = X.shape[1]
    r_s, r_l = U.shape[1], A.shape[1]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    qw, Wq = _weight_dgrad(W_res, qw, weight_blk)
    dYd = bf16_to_f64(dY)
    if _grad_bits(precision) == 16:
        qdy = None
        dYq = dYd[rows]
    else:
        qdy = quantize_1x16(dY, amax_dy)
        dYq = dequant_1x16(qdy[0], qdy[1], qdy[2], M, N)[rows]
    Pg = _lowrank_down(dYd, V, B, s)
    Pgd = bf16_to_f64(Pg)
    LR = np.concatenate([bf16_to_f64(U), bf16_to_f64(A)], axis=1)  # [K, r_s + r_l]
    dX = dYq @ Wq + Pgd[rows] @ LR.T
    P_lora = bf16_to_f64(np.asarray(P)[:, r_s:r_s + r_l])
    Pg_lora = Pgd[:, r_s:r_s + r_l]
    dB = dYd.T @ P_lora
    dA = bf16_to_f64(X).T @ Pg_lora
    return {"dX": dX, "dA": dA, "dB": dB, "Pg": Pg, "qdy": qdy, "rows": rows}


# -------------------------------------------------------------- MLP fusion
_GELU_TABLE = None


def gelu_bf16(y: np.ndarray) -> np.ndarray:
    """GELU of bf16 values, rounded once to bf16 (RNE): for each bf16 bit
    pattern y, h = bf16(0.5 y erfc(-y / sqrt 2)) from float64 (the erfc form
    stays accurate where 1 + erf would cancel, y << 0).  A bf16 input takes
    one of 65536 values, so the function is a table over every bit pattern
    (pinned against a 50-digit evaluation).  GELU is the activation between
    a DiT block's MLP linears (FourTune page, section 3.3, MLP fusion)."""
    global _GELU_TABLE
    if _GELU_TABLE is None:
        import math
        v = bf16_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))
        out = np.empty(65536, np.float64)
        for i, x in enumerate(v):
            out[i] = 0.5 * x * math.erfc(-x / math.sqrt(2.0)) if np.isfinite(x) else x
        t = bf16_from_f64(out)
        # A float64 result exactly halfway between two bf16 values arises
        # only for subnormal y, where it is y / 2 with the y^2 / sqrt(2 pi)
        # term rounded away; the true value lies above it (GELU(y) - y / 2 =
        # y (Phi(y) - 1/2) > 0 for y != 0), so such a tie rounds up.
        lo = bf16_to_f64(t)
        up = bf16_to_f64(((t.astype(np.int32) + np.where(lo >= 0, 1, -1)) & 0xFFFF).astype(np.uint16))
        tie = np.isfinite(out) & (out != lo) & (np.abs(out - lo) == np.abs(up - out)) & (up > lo)
        t[tie] = bf16_from_f64(up[tie])
        _GELU_TABLE = t
    return _GELU_TABLE[np.asarray(y, np.uint16)]


def mlp_fwd(X, up: dict, down: dict, amax_h: float, amax_x=None):
    """Forward of a DiT MLP whose two linears are triple-branch layers, with
    the FC1 GEMM fused with the FC2 quantization (FourTune page, section 3.3,
    "MLP Fusion"): Y_up = the up layer's Eq. 2 output rounded to bf16, H =
    GELU(Y_up) rounded to bf16, and the down layer's forward on H, whose
    NVFP4 tensor scale comes from the supplied amax_h (the fused kernel
    quantizes H as the tiles leave the FC1 GEMM, before the whole of H
    exists, so the tensor amax cannot come from H itself).  Every step is
    row-local given amax_x (the tensor amax of X, else X's own) and amax_h,
    so X may be a sample of token rows.  up / down: dicts of W_res, U, V, A,
    B, s and optionally qw (the 16x16 quantization of W_res).  Returns Y_up
    (bf16), H (bf16), P_up, P_down (bf16), qh = (codes, scales, g) of Q(H)
    and Y (float64) of the down layer."""
    f_up = linear_fwd(X, up["W_res"], up["U"], up["V"], up["A"], up["B"], up["s"], amax_x=amax_x,
                      qw=up.get("qw"))
    Y_up = bf16_from_f64(f_up["Y"])
    H = gelu_bf16(Y_up)
    f_dn = linear_fwd(H, down["W_res"], down["U"], down["V"], down["A"], down["B"], down["s"], amax_x=amax_h,
                      qw=down.get("qw"))
    return {"Y_up": Y_up, "H": H, "P_up": f_up["P"], "P_down": f_dn["P"], "qh": f_dn["qx"], "Y": f_dn["Y"]}


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    """||a - b||_F / ||b||_F (0 when both are zero)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    na = np.linalg.norm(a - b)
    if nb == 0.0:
        return 0.0 if na == 0.0 else float("inf")
    return float(na / nb)
