"""Ordering of back-to-back calls on one stream and one workspace.

The library's kernels are launched with programmatic stream serialization:
each may start while the previous kernel on the stream drains, and either
waits for that kernel's completion (griddepcontrol.wait) or for a counter
that the quantizer's CTAs release after their last write.  A kernel that
waited on a counter must still complete after the kernel it overlapped, or
the next call's quantizer could rewrite the workspace's Q(dY) codes and scales
while a dgrad GEMM still reads them, or a caller's copy could read a dX that
is not finished.  These tests enqueue many calls without any host
synchronisation, each with its own inputs (so an operand overwritten too
early changes a result), and compare every output bit for bit with the same
calls run one at a time with a device synchronisation after each.
"""
import dataclasses

import numpy as np
import pytest
import torch

import ft_synth
import oracle
import bit_quantized_lora_b200 as ft
from gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def _layer(shape, seed):
    inp = ft_synth.make_inputs(shape, seed)
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    return ft.prepare_layer(W_res=dev_bf16(Wr), U=dev_bf16(U), V=dev_bf16(V), A=dev_bf16(inp["A"]),
                            B=dev_bf16(inp["B"]), s=inp["s"])


def _batches(shape, n, seed):
    out = []
    for i in range(n):
        inp = ft_synth.make_inputs(shape, seed + 1000 * (i + 1))
        out.append((dev_bf16(inp["X"]), dev_bf16(inp["dY"])))
    return out


def _run(layer, batches, iters, sync_each):
    ws = ft.Workspace()
    outs = []
    for i in range(iters):
        X, dY = batches[i % len(batches)]
        Y, P = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32, ws=ws)
        if sync_each:
            torch.cuda.synchronize()
        dX, dA, dB = ft.ft_linear_bwd(layer, dY, X, P, out_dtype=ft.F32, ws=ws)
        if sync_each:
            torch.cuda.synchronize()
        outs.append((Y, P, dX, dA, dB))
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    return outs


@pytest.mark.parametrize("case", ["tiny", "tiny_m37", "tiny_m300", "attn_m37", "down_m300"])
def test_back_to_back_fwd_bwd_match_synchronised_calls(case):
    """20 forward + backward passes on one workspace with no host
    synchronisation in between.  Small token counts give the GEMMs a grid of
    one or a few CTAs, so the adapter-gradient kernel runs beside the dgrad
    GEMM and ends first (the MLP down-projection's dgrad, [300, 12288] out of
    K = 12288 contraction steps of N = 3072, runs much longer than its
    adapter gradients)."""
    base = {"tiny": (ft_synth.TINY, None), "tiny_m37": (ft_synth.TINY, 37),
            "tiny_m300": (ft_synth.TINY, 300), "attn_m37": (ft_synth.ATTN, 37),
            "down_m300": (ft_synth.MLP_DOWN, 300)}[case]
    shape = base[0] if base[1] is None else dataclasses.replace(base[0], M=base[1])
    layer = _layer(shape, 60)
    batches = _batches(shape, 4, 61)
    ref = _run(layer, batches, 4, sync_each=True)
    got = _run(layer, batches, 20, sync_each=False)
    for i, outs in enumerate(got):
        for a, b in zip(outs, ref[i % 4]):
            assert torch.equal(a, b), f"iteration {i}"


def test_mlp_backward_chain_on_default_workspace():
    """The backward of an MLP pair as a training step runs it: the
    down-projection's backward, then the up-projection's backward taking the
    first call's dX as its output gradient, on the default workspace, twice
    in a row without synchronisation; bit for bit equal to the same calls
    with a device synchronisation after each."""
    up = dataclasses.replace(ft_synth.MLP_UP, r_l=64)
    down = ft_synth.MLP_DOWN
    L_up, L_dn = _layer(up, 70), _layer(down, 71)
    inp_up, inp_dn = ft_synth.make_inputs(up, 72), ft_synth.make_inputs(down, 73)
    X_up, X_dn, dY_dn = dev_bf16(inp_up["X"]), dev_bf16(inp_dn["X"]), dev_bf16(inp_dn["dY"])
    dY_dn2 = dev_bf16(ft_synth.make_inputs(down, 74)["dY"])
    _, P_up = ft.ft_linear_fwd(L_up, X_up)
    _, P_dn = ft.ft_linear_fwd(L_dn, X_dn)
    torch.cuda.synchronize()

    def chain(sync_each):
        outs = []
        for g in (dY_dn, dY_dn2):
            dH, dA2, dB2 = ft.ft_linear_bwd(L_dn, g, X_dn, P_dn)
            if sync_each:
                torch.cuda.synchronize()
            dX, dA1, dB1 = ft.ft_linear_bwd(L_up, dH, X_up, P_up)
            if sync_each:
                torch.cuda.synchronize()
            outs.append((dH, dA2, dB2, dX, dA1, dB1))
        torch.cuda.synchronize()
        assert ft.ft_device_error() == 0
        return outs

    ref = chain(True)
    for _ in range(3):
        got = chain(False)
        for o, r in zip(got, ref):
            for a, b in zip(o, r):
                assert torch.equal(a, b)
    # the chain is not trivially constant: the two output gradients differ
    assert not torch.equal(ref[0][3], ref[1][3])
    assert np.isfinite(ref[1][3].float().cpu().numpy()).all()
