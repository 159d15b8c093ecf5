"""The DiT linear stack (the four triple-branch linears of a block: QKV
[9216, 3072], attention out [3072, 3072], MLP up [12288, 3072], MLP down
[3072, 12288]; 4608 tokens, stabilizer and LoRA rank 32) through the stack
driver, against the CPU oracle.

Per linear, run one call at a time so the workspace still holds the call's
quantized operand: Q(X) after the forward and Q(dY) after the backward equal
the oracle's codes, scales and tensor scale bit for bit on the full tensors
(integer work); Y and dX match the FP64 oracle on 256 sampled token rows and
dA, dB on all rows within relative Frobenius error 1e-3 (FP32 output mode);
every entry of P and Pg is within one bf16 rounding plus the FP32 summation
bound.  Then the block's whole step -- the four forwards, then the four
backwards in reverse order, enqueued without synchronisation on one
workspace -- reproduces those outputs bit for bit."""
import numpy as np
import pytest
import torch

import ft_synth
import oracle
import bit_quantized_lora_b200 as ft
from bit_quantized_lora_b200.stack import LinearStack
from gpu_util import check_lowrank_down, dev_bf16, host, host_u16

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _ws_qact(ws, M, L, C):
    co, so, go = ft.ft_workspace_qact(M, L.N, L.K, L.r_s, L.r_l)
    raw = ws.buf
    codes = host(raw[co:co + M * C // 2]).reshape(M, C // 2)
    scales = host(raw[so:so + M * C // 16]).reshape(M, C // 16)
    g = host(raw[go:go + 4]).view(np.float32)[0]
    return codes, scales, g


def test_dit_block_linears_against_the_oracle():
    shapes = ft_synth.dit_block_linears(0)
    M = shapes[0].M
    inps, splits, layers = [], [], []
    for j, sh in enumerate(shapes):
        inp = ft_synth.make_inputs(sh, seed=100 + j)
        U, V, Wr = oracle.svd_split(inp["W"], sh.r_s)
        inps.append(inp)
        splits.append((U, V, Wr))
        layers.append(ft.prepare_layer(W_res=dev_bf16(Wr), U=dev_bf16(U), V=dev_bf16(V), A=dev_bf16(inp["A"]),
                                       B=dev_bf16(inp["B"]), s=inp["s"]))
    st = LinearStack(layers, M, "cuda", out_dtype=ft.F32)
    Xs = [dev_bf16(i["X"]) for i in inps]
    dYs = [dev_bf16(i["dY"]) for i in inps]
    rows = np.sort(np.random.default_rng(5).choice(M, 256, replace=False))
    ref_out = []
    for j, (sh, inp, (U, V, Wr), L) in enumerate(zip(shapes, inps, splits, layers)):
        st.forward_layer(j, Xs[j])
        torch.cuda.synchronize()
        assert ft.ft_device_error() == 0
        codes, scales, g = _ws_qact(st.ws, M, L, L.K)
        qw = oracle.quantize_16x16(Wr)
        f = oracle.linear_fwd(inp["X"], Wr, U, V, inp["A"], inp["B"], inp["s"], rows=rows, qw=qw)
        rc, rs, rg = f["qx"]
        assert np.float32(g) == np.float32(rg), sh.name
        np.testing.assert_array_equal(scales, rs)
        np.testing.assert_array_equal(codes, rc)
        b = st.bufs[j]
        assert oracle.rel_fro(host(b.Y)[rows], f["Y"]) <= TOL, sh.name
        check_lowrank_down(host_u16(b.P), f["P"], oracle.bf16_to_f64(inp["X"]), oracle.bf16_to_f64(U),
                           oracle.bf16_to_f64(inp["A"]), inp["s"])

        st.backward_layer(j, dYs[j], Xs[j])
        torch.cuda.synchronize()
        assert ft.ft_device_error() == 0
        codes, scales, g = _ws_qact(st.ws, M, L, L.N)
        bw = oracle.linear_bwd(inp["dY"], inp["X"], Wr, U, V, inp["A"], inp["B"], inp["s"], f["P"], rows=rows,
                               qw=qw)
        rc, rs, rg = bw["qdy"]
        assert np.float32(g) == np.float32(rg), sh.name
        np.testing.assert_array_equal(scales, rs)
        np.testing.assert_array_equal(codes, rc)
        assert oracle.rel_fro(host(b.dX)[rows], bw["dX"]) <= TOL, sh.name
        assert oracle.rel_fro(host(b.dA), bw["dA"]) <= TOL, sh.name
        assert oracle.rel_fro(host(b.dB), bw["dB"]) <= TOL, sh.name
        ref_out.append([t.clone() for t in (b.Y, b.P, b.dX, b.dA, b.dB)])

    # the block as one step: forwards in order, backwards in reverse order,
    # no synchronisation in between; the same bits as the calls one by one
    for t in (st.grads,) + tuple(x for b in st.bufs for x in (b.Y, b.dX)):
        t.fill_(float("nan"))
    st.step(Xs, dYs)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    for j, b in enumerate(st.bufs):
        for a, r in zip((b.Y, b.P, b.dX, b.dA, b.dB), ref_out[j]):
            assert torch.equal(a, r), shapes[j].name
