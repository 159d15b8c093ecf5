"""Seeded synthetic inputs for the W4A4G4 triple-branch linear layer.

This module only draws random tensors and rounds them to bf16; it holds none
of the layer's arithmetic (no quantization, no SVD split, no products).  It is
the one module that both the CUDA path's tests/bench and the CPU oracle read.

Shapes stand in for FLUX.1-dev at 1024x1024 (4096 image + 512 text tokens,
hidden 3072, MLP 12288), the scale the FourTune page reports on; no FLUX
weights or datasets are used.

Recipe (numpy PCG64, ``default_rng(seed)``, seed = workload index; values drawn
in float64 then rounded to bf16 with round-to-nearest-even; draw order X, W,
A, B, dY):
  tiny   M=128  K=256   N=256   r_s=16 r_l=16  X~N(0,1), 4 channels x50;
                                               W~N(0,0.02^2)
  attn   M=4608 K=3072  N=3072  r_s=32 r_l=16  X~N(0,1), 1% channels x30;
                                               W~N(0,0.02^2)
  mlp_up M=4608 K=3072  N=12288 r_s=32 r_l=32  as attn
  mlp_dn M=4608 K=12288 N=3072  r_s=32 r_l=64  X=GELU_erf(N(0,1));
                                               W~N(0,0.01^2);
                                               dY=1e-3*StudentT(nu=3)
  dit8   8 blocks x {qkv 9216x3072, out 3072x3072, up 12288x3072,
                     down 3072x12288}, r_s=r_l=32, M=4608
All: A~N(0,0.01^2) [K,r_l], B~N(0,0.01^2) [N,r_l], s=1, dY~N(0,1) unless
stated.  The outlier channels are columns of X chosen by the generator.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class LinearShape:
    name: str
    M: int
    K: int
    N: int
    r_s: int
    r_l: int
    x_kind: str = "normal_outliers"   # or "gelu"
    outlier_channels: int = 0          # number of amplified columns of X
    outlier_factor: float = 1.0
    w_std: float = 0.02
    dy_kind: str = "normal"            # or "student_t3"
    s: float = 1.0


TINY = LinearShape("tiny", 128, 256, 256, 16, 16, outlier_channels=4, outlier_factor=50.0)
ATTN = LinearShape("attn_proj", 4608, 3072, 3072, 32, 16, outlier_channels=31, outlier_factor=30.0)
MLP_UP = LinearShape("mlp_up", 4608, 3072, 12288, 32, 32, outlier_channels=31, outlier_factor=30.0)
MLP_DOWN = LinearShape("mlp_down", 4608, 12288, 3072, 32, 64, x_kind="gelu", w_std=0.01,
                       dy_kind="student_t3")

WORKLOADS = {0: TINY, 1: ATTN, 2: MLP_UP, 3: MLP_DOWN}


def dit_block_linears(block: int) -> list[LinearShape]:
    """The four triple-branch linears of one DiT block (hidden 3072, 24 heads,
    MLP 12288), batch 1 x 4608 tokens, r_s = r_l = 32."""
    return [
        LinearShape(f"b{block}.qkv", 4608, 3072, 9216, 32, 32, outlier_channels=31, outlier_factor=30.0),
        LinearShape(f"b{block}.out", 4608, 3072, 3072, 32, 32, outlier_channels=31, outlier_factor=30.0),
        LinearShape(f"b{block}.up", 4608, 3072, 12288, 32, 32, outlier_channels=31, outlier_factor=30.0),
        LinearShape(f"b{block}.down", 4608, 12288, 3072, 32, 32, x_kind="gelu", w_std=0.01,
                    dy_kind="student_t3"),
    ]


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns, round-to-nearest-even (input generation)."""
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    q = np.maximum(e - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(v, -q)), q)
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _gelu_erf(x: np.ndarray) -> np.ndarray:
    from scipy.special import erf
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def make_inputs(shape: LinearShape, seed: int, M: int | None = None) -> dict:
    """Draw X, W, A, B, dY (bf16 bit patterns, uint16) for one linear.

    M overrides the token count (e.g. a per-rank shard); the draw order is
    fixed so a given (shape, seed, M) always gives the same tensors.
    """
    rng = np.random.default_rng(seed)
    M = shape.M if M is None else M
    K, N = shape.K, shape.N
    if shape.x_kind == "gelu":
        X = _gelu_erf(rng.standard_normal((M, K)))
    else:
        X = rng.standard_normal((M, K))
        if shape.outlier_channels:
            cols = rng.choice(K, size=shape.outlier_channels, replace=False)
            X[:, cols] *= shape.outlier_factor
    W = rng.standard_normal((N, K)) * shape.w_std
    A = rng.standard_normal((K, shape.r_l)) * 0.01
    B = rng.standard_normal((N, shape.r_l)) * 0.01
    if shape.dy_kind == "student_t3":
        dY = 1e-3 * rng.standard_t(3, size=(M, N))
    else:
        dY = rng.standard_normal((M, N))
    return {
        "X": to_bf16_bits(X),
        "W": to_bf16_bits(W),
        "A": to_bf16_bits(A),
        "B": to_bf16_bits(B),
        "dY": to_bf16_bits(dY),
        "s": float(shape.s),
    }


def lossless_fp4_operand(rng: np.random.Generator, rows: int, cols: int, block_rows: int,
                         exp_range=(-2, 2)) -> np.ndarray:
    """bf16 matrix whose every block (block_rows x 16) holds E2M1 grid values
    times one power of two and contains a +-6 element, so that block
    quantization with any power-of-two tensor scale is lossless."""
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    v = grid[rng.integers(0, 8, size=(rows, cols))] * rng.choice([-1.0, 1.0], size=(rows, cols))
    for i in range(0, rows, block_rows):
        for j in range(0, cols, 16):
            e = rng.integers(exp_range[0], exp_range[1] + 1)
            blk = v[i:i + block_rows, j:j + 16]
            blk[0, 0] = 6.0 * rng.choice([-1.0, 1.0])
            v[i:i + block_rows, j:j + 16] = blk * (2.0 ** e)
    return to_bf16_bits(v)
