"""The 4-bit GEMM on CTA pairs (ft_set_gemm_mode): pairs of CTAs on the two
SMs of a TPC share 256 x 256 output tiles.  It computes the same sums as the
one-CTA tiling, so Y, dX and the fused MLP's H and Q(H) must be identical
bit for bit between the two modes; the other GPU tests check the default
(pair) mode against the oracle.

Cases cover a ragged pair tile whose second CTA lies wholly past the rows
(M = 300: rows 256..299 and an empty half), a single spare row (M = 129),
the rank variants (no low-rank term; 16 + 112 over two atoms; 64 + 64) and
the fused MLP forward.
"""
import numpy as np
import pytest
import torch

import ft_synth
import oracle
import bit_quantized_lora_b200 as ft
from gpu_util import dev_bf16, scalar_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _default_mode():
    yield
    ft.ft_set_gemm_mode(ft.GEMM_PAIRS)


def _layer(shape, seed):
    inp = ft_synth.make_inputs(shape, seed)
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    layer = ft.prepare_layer(W_res=dev_bf16(Wr), U=dev_bf16(U), V=dev_bf16(V), A=dev_bf16(inp["A"]),
                             B=dev_bf16(inp["B"]), s=inp["s"])
    return inp, layer


def _fwd_bwd(layer, X, dY, mode):
    ft.ft_set_gemm_mode(mode)
    Y, P = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32)
    dX, dA, dB = ft.ft_linear_bwd(layer, dY, X, P, out_dtype=ft.F32)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    return Y, P, dX, dA, dB


@pytest.mark.parametrize("M,r_s,r_l", [(129, 32, 32), (300, 32, 32), (1000, 32, 16), (512, 0, 0),
                                       (384, 16, 112), (640, 64, 64)])
def test_pairs_match_single_cta_tiles(M, r_s, r_l):
    shape = ft_synth.LinearShape("pairs", M, 512, 768, r_s, r_l, outlier_channels=4, outlier_factor=20.0)
    inp, layer = _layer(shape, 71)
    X, dY = dev_bf16(inp["X"]), dev_bf16(inp["dY"])
    a = _fwd_bwd(layer, X, dY, ft.GEMM_SINGLE)
    b = _fwd_bwd(layer, X, dY, ft.GEMM_PAIRS)
    for x, y in zip(a, b):
        if x is None:
            assert y is None
        else:
            assert torch.equal(x, y)
    assert np.isfinite(a[0].cpu().numpy()).all()


def test_pairs_match_single_cta_tiles_attention_shape():
    shape = ft_synth.ATTN
    inp, layer = _layer(shape, 72)
    X, dY = dev_bf16(inp["X"]), dev_bf16(inp["dY"])
    a = _fwd_bwd(layer, X, dY, ft.GEMM_SINGLE)
    b = _fwd_bwd(layer, X, dY, ft.GEMM_PAIRS)
    assert torch.equal(a[0], b[0]) and torch.equal(a[2], b[2])


@pytest.mark.parametrize("M", [300, 1024])
def test_pairs_match_single_cta_tiles_fused_mlp(M):
    up_shape = ft_synth.LinearShape("mlp_up", M, 256, 512, 16, 16, outlier_channels=4, outlier_factor=20.0)
    dn_shape = ft_synth.LinearShape("mlp_dn", M, 512, 256, 16, 32, w_std=0.05)
    up_inp, up = _layer(up_shape, 73)
    _, down = _layer(dn_shape, 74)
    X = dev_bf16(up_inp["X"])
    # Q(H) as the fused epilogue leaves it in the down layer's workspace
    base = (ft.ft_workspace_bytes(M, up.N, up.K, up.r_s, up.r_l) + 255) // 256 * 256
    co, so, _ = ft.ft_workspace_qact(M, down.N, down.K, down.r_s, down.r_l)
    outs = []
    for mode in (ft.GEMM_SINGLE, ft.GEMM_PAIRS):
        ft.ft_set_gemm_mode(mode)
        ws = ft.Workspace()
        Y, H, P_up, P_down = ft.ft_mlp_fwd(up, down, X, scalar_dev(4.0), out_dtype=ft.F32, ws=ws)
        torch.cuda.synchronize()
        assert ft.ft_device_error() == 0
        codes = ws.buf[base + co:base + co + M * down.K // 2].clone()
        scales = ws.buf[base + so:base + so + M * down.K // 16].clone()
        outs.append((Y, H, P_up, P_down, codes, scales))
    for x, y in zip(outs[0], outs[1]):
        assert torch.equal(x, y)
