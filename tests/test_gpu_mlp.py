"""MLP fusion (FourTune page, section 3.3): FC1's GEMM applies GELU in its
epilogue and quantizes its output for FC2 as the tiles leave.

Checks, through the C ABI:
  * the GELU itself: every finite bf16 input through ft_gelu_bf16 equals the
    oracle's once-rounded GELU bit for bit (65536 values);
  * the fused forward: H equals the oracle's GELU of the plain FC1 call's
    bf16 output bit for bit (the same GEMM computes the same FP32 values);
    Q(H), read back from the workspace, equals the oracle's quantization of
    H with the supplied tensor amax bit for bit (also an amax below max|H|,
    which saturates); P_up equals the plain call's; P_down is within one
    bf16 rounding plus the FP32 summation bound of the oracle's; Y matches
    the oracle's down layer on H within 1e-3 relative Frobenius error and
    every sampled entry within its FP32 summation bound.
"""
import dataclasses

import numpy as np
import pytest
import torch

import ft_synth
import oracle
import bit_quantized_lora_b200 as ft
from gpu_util import check_fp32_sum_bound, check_lowrank_down, dev_bf16, host, host_u16, scalar_dev

pytestmark = pytest.mark.gpu

TOL = 1e-3


def test_gelu_every_finite_bf16_value():
    u = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = np.isfinite(oracle.bf16_to_f64(u))
    y = u[finite]
    y = np.concatenate([y, np.zeros((-len(y)) % 8, np.uint16)])
    h = ft.ft_gelu_bf16(dev_bf16(y.reshape(1, -1)))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_u16(h).ravel(), oracle.gelu_bf16(y))


def _layer(shape, seed):
    inp = ft_synth.make_inputs(shape, seed)
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    layer = ft.prepare_layer(W_res=dev_bf16(Wr), U=dev_bf16(U), V=dev_bf16(V), A=dev_bf16(inp["A"]),
                             B=dev_bf16(inp["B"]), s=inp["s"])
    return inp, dict(W_res=Wr, U=U, V=V, A=inp["A"], B=inp["B"], s=inp["s"]), layer


def _q_h(ws, M, up, down):
    base = (ft.ft_workspace_bytes(M, up.N, up.K, up.r_s, up.r_l) + 255) // 256 * 256
    co, so, go = ft.ft_workspace_qact(M, down.N, down.K, down.r_s, down.r_l)
    raw = ws.buf
    C = down.K
    codes = host(raw[base + co:base + co + M * C // 2]).reshape(M, C // 2)
    scales = host(raw[base + so:base + so + M * C // 16]).reshape(M, C // 16)
    g = host(raw[base + go:base + go + 4]).view(np.float32)[0]
    return codes, scales, g


@pytest.mark.parametrize("case", ["tiny", "tiny_ragged", "tiny_saturating", "dit"])
def test_fused_mlp_forward(case):
    if case == "dit":
        up_shape, dn_shape = ft_synth.dit_block_linears(0)[2], ft_synth.dit_block_linears(0)[3]
        M = up_shape.M
    else:
        M = 300 if case == "tiny_ragged" else 128
        up_shape = ft_synth.LinearShape("mlp_up", M, 256, 512, 16, 16, outlier_channels=4, outlier_factor=20.0)
        dn_shape = ft_synth.LinearShape("mlp_dn", M, 512, 256, 16, 32, w_std=0.05)
    up_inp, up_o, up = _layer(up_shape, 31)
    _, dn_o, down = _layer(dn_shape, 32)
    X = dev_bf16(up_inp["X"])
    # the plain FC1 call and its bf16 output: the fused epilogue's input
    Y_up, P_up_ref = ft.ft_linear_fwd(up, X)
    torch.cuda.synchronize()
    H_ref = oracle.gelu_bf16(host_u16(Y_up))
    amax_true = float(np.abs(oracle.bf16_to_f64(H_ref)).max())
    amax_h = amax_true * (0.5 if case == "tiny_saturating" else 1.0)
    ws = ft.Workspace()
    Y, H, P_up, P_down = ft.ft_mlp_fwd(up, down, X, scalar_dev(amax_h), out_dtype=ft.F32, ws=ws)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    np.testing.assert_array_equal(host_u16(H), H_ref)
    assert torch.equal(P_up, P_up_ref)
    codes, scales, g = _q_h(ws, M, up, down)
    rc, rs, rg = oracle.quantize_1x16(H_ref, amax_h)
    assert np.float32(g) == np.float32(rg)
    np.testing.assert_array_equal(scales, rs)
    np.testing.assert_array_equal(codes, rc)
    # the down layer on H: P_down and Y against the oracle
    rows = np.arange(M) if case != "dit" else np.sort(np.random.default_rng(9).choice(M, 256, replace=False))
    qw = oracle.quantize_16x16(dn_o["W_res"])
    f = oracle.linear_fwd(H_ref, dn_o["W_res"], dn_o["U"], dn_o["V"], dn_o["A"], dn_o["B"], dn_o["s"], rows=rows,
                          amax_x=amax_h, qw=qw)
    d = oracle.bf16_to_f64
    check_lowrank_down(host_u16(P_down), f["P"], d(H_ref), d(dn_o["U"]), d(dn_o["A"]), dn_o["s"])
    Yg = host(Y)[rows]
    assert oracle.rel_fro(Yg, f["Y"]) <= TOL, oracle.rel_fro(Yg, f["Y"])
    Hq = oracle.dequant_1x16(rc, rs, rg, M, down.K)[rows]
    Wq = oracle.dequant_16x16(qw[0], qw[2], qw[3], down.N, down.K)
    LR = np.concatenate([d(dn_o["V"]), d(dn_o["B"])], axis=1)
    Pd = d(host_u16(P_down))[rows]
    check_fp32_sum_bound(Yg, Hq @ Wq.T + Pd @ LR.T, np.abs(Hq) @ np.abs(Wq).T + np.abs(Pd) @ np.abs(LR).T, down.K)
    if case == "dit":
        # the same kernels quantize H and project it down in the unfused call
        # with the same tensor amax: Y is bit-identical
        Y2, P2 = ft.ft_linear_fwd(down, H, amax_x=scalar_dev(amax_h), out_dtype=ft.F32)
        torch.cuda.synchronize()
        assert torch.equal(P2, P_down) and torch.equal(Y2, Y)
        # and against the oracle's whole fused MLP on the sampled rows
        m = oracle.mlp_fwd(np.ascontiguousarray(up_inp["X"][rows]), dict(up_o, qw=oracle.quantize_16x16(up_o["W_res"])),
                           dict(dn_o, qw=qw), amax_h, amax_x=oracle.amax_bf16(up_inp["X"]))
        assert oracle.rel_fro(Yg, m["Y"]) <= TOL


def test_fused_mlp_reports_amax_of_h_for_delayed_scaling():
    """amax_h_out = max|H| exactly (FC1's epilogue); passed back as amax_h
    (the next step's tensor scale) it quantizes H as the oracle does with the
    true amax."""
    M = 300
    up_shape = ft_synth.LinearShape("mlp_up", M, 256, 512, 16, 16, outlier_channels=4, outlier_factor=20.0)
    dn_shape = ft_synth.LinearShape("mlp_dn", M, 512, 256, 16, 32, w_std=0.05)
    up_inp, _, up = _layer(up_shape, 41)
    _, _, down = _layer(dn_shape, 42)
    X = dev_bf16(up_inp["X"])
    am = torch.zeros(1, dtype=torch.float32, device="cuda")
    _, H, _, _ = ft.ft_mlp_fwd(up, down, X, scalar_dev(1.0), ws=ft.Workspace(), amax_h_out=am)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    H_host = host_u16(H)
    true_amax = float(np.abs(oracle.bf16_to_f64(H_host)).max())
    assert am.item() == true_amax
    ws = ft.Workspace()
    _, H2, _, _ = ft.ft_mlp_fwd(up, down, X, am.clone(), ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(H2, H)
    codes, scales, g = _q_h(ws, M, up, down)
    rc, rs, rg = oracle.quantize_1x16(H_host, true_amax)
    assert np.float32(g) == np.float32(rg)
    np.testing.assert_array_equal(scales, rs)
    np.testing.assert_array_equal(codes, rc)
