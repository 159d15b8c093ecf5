"""ctypes declarations of the C ABI in include/ft.h.  Loading fails loudly when
the CUDA library has not been built: there is no fallback implementation."""
from __future__ import annotations

import ctypes
import os

from . import build as _build

c_i64 = ctypes.c_int64
c_vp = ctypes.c_void_p


class FtFp4(ctypes.Structure):
    _fields_ = [
        ("codes", c_vp),
        ("scales", c_vp),
        ("tscale", c_vp),
        ("rows", c_i64),
        ("cols", c_i64),
        ("blk", ctypes.c_int),
    ]


class FtLinear(ctypes.Structure):
    _fields_ = [
        ("N", c_i64),
        ("K", c_i64),
        ("r_s", c_i64),
        ("r_l", c_i64),
        ("s", ctypes.c_float),
        ("w_k", FtFp4),
        ("w_n", FtFp4),
        ("U", c_vp),
        ("V", c_vp),
        ("A", c_vp),
        ("B", c_vp),
        ("op_k", c_vp),
        ("op_n", c_vp),
        ("precision", ctypes.c_int32),
        ("wd_k", c_vp),
        ("wd_n", c_vp),
    ]


# name -> (restype, argtypes), exactly the declarations of include/ft.h
SIGNATURES = {
    "ft_quantize": (ctypes.c_int, [c_vp, c_i64, c_i64, c_i64, ctypes.c_int, c_vp,
                                   ctypes.POINTER(FtFp4), c_vp, ctypes.c_size_t, c_vp]),
    "ft_quantize_transpose": (ctypes.c_int, [c_vp, c_i64, c_i64, c_i64, ctypes.c_int, c_vp,
                                             ctypes.POINTER(FtFp4), ctypes.POINTER(FtFp4), c_vp,
                                             ctypes.c_size_t, c_vp]),
    "ft_linear_fwd": (ctypes.c_int, [ctypes.POINTER(FtLinear), c_vp, c_i64, c_vp, c_vp, ctypes.c_int,
                                     c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp]),
    "ft_linear_bwd": (ctypes.c_int, [ctypes.POINTER(FtLinear), c_vp, c_vp, c_vp, c_i64, c_vp, c_vp,
                                     ctypes.c_int, c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp]),
    "ft_dequant_weight_operands": (ctypes.c_int, [ctypes.POINTER(FtFp4), ctypes.POINTER(FtFp4), c_vp, c_vp,
                                                  c_vp]),
    "ft_gelu_bf16": (ctypes.c_int, [c_vp, c_vp, c_i64, c_vp]),
    "ft_mlp_fwd": (ctypes.c_int, [ctypes.POINTER(FtLinear), ctypes.POINTER(FtLinear), c_vp, c_i64, c_vp, c_vp,
                                  c_vp, c_vp, ctypes.c_int, c_vp, c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp]),
    "ft_mlp_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(FtLinear), ctypes.POINTER(FtLinear), c_i64]),
    "ft_workspace_bytes": (ctypes.c_size_t, [c_i64, c_i64, c_i64, c_i64, c_i64]),
    "ft_quantize_workspace_bytes": (ctypes.c_size_t, []),
    "ft_weight_operand_bytes": (ctypes.c_size_t, [c_i64, c_i64]),
    "ft_pack_weight_operands": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_vp]),
    "ft_pack_weight_operands_1x16": (ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_vp]),
    "ft_workspace_qact": (ctypes.c_int, [c_i64, c_i64, c_i64, c_i64, c_i64,
                                         ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t),
                                         ctypes.POINTER(ctypes.c_size_t)]),
    "ft_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int), c_vp]),
    "ft_set_cooperative_quantizer": (ctypes.c_int, [ctypes.c_int]),
    "ft_set_gemm_mode": (ctypes.c_int, [ctypes.c_int]),
    "ft_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "ft_linear_fwd_noalloc": (ctypes.c_int, [ctypes.POINTER(FtLinear), c_vp, c_i64, c_vp, c_vp,
                                             ctypes.c_int, c_vp, c_vp]),
    "ft_linear_fwd_noalloc_max_bytes": (ctypes.c_size_t, []),
    "ft_timing_enable": (ctypes.c_int, [ctypes.c_int]),
    "ft_timing_read": (ctypes.c_int, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                      ctypes.POINTER(c_i64)]),
    "ft_timing_reset": (ctypes.c_int, []),
}

_lib = None


def lib_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True):
    """Load libft_b200.so (building it first if it is missing or stale and
    nvcc is available).  Raises if the library cannot be loaded."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if build_if_missing and _build.needs_build():
        _build.build()
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing; run python -m bit_quantized_lora_b200.build")
    L = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


class FtError(RuntimeError):
    def __init__(self, name: str, status: int):
        msg = load().ft_status_str(status).decode()
        super().__init__(f"{name} failed: {msg} ({status})")
        self.status = status


def check(name: str, status: int) -> None:
    if status != 0:
        raise FtError(name, status)
