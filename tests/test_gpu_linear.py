"""GPU parity of the triple-branch linear (forward Eq. 2, backward Eq. 3 and
the adapter gradients) against the CPU oracle.

Bar: Y, dX, dA, dB within relative Frobenius error 1e-3 of the FP64 oracle
(FP32 output mode), and every entry within the FP32 summation error bound of
its reference on the same operands; exactly equal when every operand is losslessly
representable (the FP4 GEMM then has an exact FP32 result); each entry of P
within one bf16 rounding plus the FP32 summation error bound of its
reference; the BF16 output mode within one bf16 ulp of the rounded oracle;
the device error word stays clear."""
import numpy as np
import pytest
import torch

import ft_synth
import oracle
import bit_quantized_lora_b200 as ft
from gpu_util import (bf16_ulp_diff, check_fp32_sum_bound, check_lowrank_down, dev_bf16, host, host_u16,
                      lossless_operand, scalar_dev, selection_factor)

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _dev_or_none(u16):
    return None if u16 is None or u16.shape[1] == 0 else dev_bf16(u16)


def _prep(shape, seed, M=None, r_s=None, r_l=None):
    if r_s is not None or r_l is not None:
        import dataclasses
        shape = dataclasses.replace(shape, r_s=shape.r_s if r_s is None else r_s,
                                    r_l=shape.r_l if r_l is None else r_l)
    inp = ft_synth.make_inputs(shape, seed, M)
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    layer = ft.prepare_layer(W_res=dev_bf16(Wr), U=_dev_or_none(U), V=_dev_or_none(V),
                             A=_dev_or_none(inp["A"]), B=_dev_or_none(inp["B"]), s=inp["s"])
    return inp, U, V, Wr, layer


def _run_and_compare(shape, seed, M=None, rows=None, r_s=None, r_l=None, bf16_check=False):
    inp, U, V, Wr, layer = _prep(shape, seed, M, r_s, r_l)
    X, dY, A, B, s = inp["X"], inp["dY"], inp["A"], inp["B"], inp["s"]
    Xd, dYd = dev_bf16(X), dev_bf16(dY)
    Y, P = ft.ft_linear_fwd(layer, Xd, out_dtype=ft.F32)
    dX, dA, dB = ft.ft_linear_bwd(layer, dYd, Xd, P, out_dtype=ft.F32)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    Mrows = X.shape[0]
    if rows is None:
        rows = np.arange(Mrows)
    qw = oracle.quantize_16x16(Wr)
    f = oracle.linear_fwd(X, Wr, U, V, A, B, s, rows=rows, qw=qw)
    b = oracle.linear_bwd(dY, X, Wr, U, V, A, B, s, f["P"], rows=rows, qw=qw)
    Yg, dXg = host(Y)[rows], host(dX)[rows]
    assert oracle.rel_fro(Yg, f["Y"]) <= TOL, oracle.rel_fro(Yg, f["Y"])
    assert oracle.rel_fro(dXg, b["dX"]) <= TOL, oracle.rel_fro(dXg, b["dX"])
    if layer.r_l > 0:
        assert oracle.rel_fro(host(dA), b["dA"]) <= TOL, oracle.rel_fro(host(dA), b["dA"])
        assert oracle.rel_fro(host(dB), b["dB"]) <= TOL, oracle.rel_fro(host(dB), b["dB"])
    if layer.r_s + layer.r_l > 0:
        check_lowrank_down(host_u16(P), f["P"], oracle.bf16_to_f64(X), oracle.bf16_to_f64(U),
                           oracle.bf16_to_f64(A), s)
    _check_elementwise(layer, inp, U, V, qw, f, b, rows, host_u16(P), host(Y), host(dX),
                       None if dA is None else host(dA), None if dB is None else host(dB))
    if bf16_check:
        # the BF16 mode rounds the same FP32 value the FP32 mode stores
        Yb, _ = ft.ft_linear_fwd(layer, Xd, out_dtype=ft.BF16)
        torch.cuda.synchronize()
        assert torch.equal(Yb, Y.to(torch.bfloat16))
        # and lies within one bf16 ulp of the rounded oracle wherever the
        # value is not a near-cancellation (|Y| above 1/64 of the rms).  A
        # row whose saved P took the other, equally valid bf16 rounding of
        # an entry (checked above) shifts by that rounding times V or B, so
        # the ulp comparison runs on the rows whose P is identical.
        same = np.all(host_u16(P)[rows] == f["P"][rows], axis=1) if P.numel() else np.ones(len(rows), bool)
        assert same.mean() > 0.5
        ref = oracle.bf16_from_f64(f["Y"])
        ulp = bf16_ulp_diff(host_u16(Yb)[rows], ref)[same]
        big = (np.abs(f["Y"]) >= np.sqrt(np.mean(f["Y"] ** 2)) / 64)[same]
        assert ulp[big].max() <= 1 and (ulp > 0).mean() < 0.01
    return layer


def _check_elementwise(layer, inp, U, V, qw, f, b, rows, P_gpu, Y, dX, dA, dB):
    """Every sampled entry of Y, dX and every entry of dA, dB within the FP32
    summation bound of its own reference (check_fp32_sum_bound).  The
    references take the operands the kernels took: the dequantized Q(X),
    Q(dY), Q(W_res) of the oracle (bit-identical to the GPU's, checked
    elsewhere) and the GPU's saved P where P is an operand (Y's low-rank
    term, dB).  Pg never leaves the workspace, so dX and dA get an
    allowance of the valid alternative roundings of Pg (one bf16 ulp plus
    Pg's own FP32 summation bound, as for P)."""
    from gpu_util import bf16_ulp_of
    X, dY, A, B, s = inp["X"], inp["dY"], inp["A"], inp["B"], inp["s"]
    N, K, r_s, r_l = layer.N, layer.K, layer.r_s, layer.r_l
    M = X.shape[0]
    d = oracle.bf16_to_f64
    Xq = oracle.dequant_1x16(*f["qx"], M, K)[rows]
    dYq = oracle.dequant_1x16(*b["qdy"], M, N)[rows]
    Wq = oracle.dequant_16x16(qw[0], qw[2], qw[3], N, K)
    Pd = d(P_gpu)
    LRf = np.concatenate([d(V), d(B)], axis=1)
    LRb = np.concatenate([d(U), d(A)], axis=1)
    ref = Xq @ Wq.T + Pd[rows] @ LRf.T
    absdot = np.abs(Xq) @ np.abs(Wq).T + np.abs(Pd[rows]) @ np.abs(LRf).T
    check_fp32_sum_bound(Y[rows], ref, absdot, K)
    Pg = d(b["Pg"])
    dYd = d(dY)
    mag = np.concatenate([np.abs(dYd) @ np.abs(d(V)), abs(s) * (np.abs(dYd) @ np.abs(d(B)))], axis=1)
    dPg = bf16_ulp_of(Pg) + N * 2.0 ** -23 * mag  # Pg's valid alternative roundings
    ref = dYq @ Wq + Pg[rows] @ LRb.T
    absdot = np.abs(dYq) @ np.abs(Wq) + np.abs(Pg[rows]) @ np.abs(LRb).T
    check_fp32_sum_bound(dX[rows], ref, absdot, N, slack=dPg[rows] @ np.abs(LRb).T)
    if r_l > 0:
        Xd = d(X)
        P_lora = Pd[:, r_s:r_s + r_l]
        check_fp32_sum_bound(dB, dYd.T @ P_lora, np.abs(dYd).T @ np.abs(P_lora), M)
        Pg_lora = Pg[:, r_s:r_s + r_l]
        check_fp32_sum_bound(dA, Xd.T @ Pg_lora, np.abs(Xd).T @ np.abs(Pg_lora), M,
                             slack=np.abs(Xd).T @ dPg[:, r_s:r_s + r_l])


@pytest.mark.parametrize("K", [256, 512, 768, 1024])
def test_lossless_operands_give_exact_fp32_gemm(K):
    """Every operand on the E2M1 grid times a power of two and a power-of-two
    tensor scale: quantization is lossless, the products are exact and the
    sums fit FP32, so forward and dgrad must equal the exact matmul."""
    rng = np.random.default_rng(40 + K)
    M, N = 256, 512
    X = ft_synth.lossless_fp4_operand(rng, M, K, 1, exp_range=(-1, 1))
    Wr = ft_synth.lossless_fp4_operand(rng, N, K, 16, exp_range=(-1, 1))
    dY = ft_synth.lossless_fp4_operand(rng, M, N, 1, exp_range=(-1, 1))
    amax = 2688.0  # g = 1
    layer = ft.prepare_layer(W_res=dev_bf16(Wr), amax=scalar_dev(amax))
    Y, _ = ft.ft_linear_fwd(layer, dev_bf16(X), amax_x=scalar_dev(amax), out_dtype=ft.F32)
    dX, _, _ = ft.ft_linear_bwd(layer, dev_bf16(dY), dev_bf16(X), torch.empty(0, device="cuda"),
                                amax_dy=scalar_dev(amax), out_dtype=ft.F32)
    torch.cuda.synchronize()
    Xf, Wf, dYf = oracle.bf16_to_f64(X), oracle.bf16_to_f64(Wr), oracle.bf16_to_f64(dY)
    np.testing.assert_array_equal(host(Y).astype(np.float64), Xf @ Wf.T)
    np.testing.assert_array_equal(host(dX).astype(np.float64), dYf @ Wf)


@pytest.mark.parametrize("case", ["attn", "mlp_up"])
def test_lossless_full_size_is_bit_exact(case):
    """Full-size workloads (4608 tokens) on operands that every step of the
    layer represents exactly: activations, gradients and the weight hold
    E2M1 grid values times a power of two per block (quantization with
    tensor scale 1 is lossless), and U, V, A, B select one input column per
    rank column with a factor +-2^k (so P, Pg and the low-rank products have
    a single exact term); s = 2.  Every sum is a multiple of 2^-4 whose
    absolute terms add up to less than 2^20, so FP32 accumulation is exact
    in any order.  Y, dX, dA, dB must then equal the exact result bit for
    bit, element by element -- every tile of the persistent GEMM (each CTA
    takes several), the low-rank epilogue's columns, the split reductions --
    and the BF16 output mode must be the exact value rounded once."""
    shape = ft_synth.ATTN if case == "attn" else ft_synth.MLP_UP
    M, N, K, r_s, r_l = shape.M, shape.N, shape.K, shape.r_s, shape.r_l
    rng = np.random.default_rng(90 if case == "attn" else 91)
    X = lossless_operand(rng, M, K, 1)
    dY = lossless_operand(rng, M, N, 1)
    Wr = lossless_operand(rng, N, K, 16)
    U, V = selection_factor(rng, K, r_s), selection_factor(rng, N, r_s)
    A, B = selection_factor(rng, K, r_l), selection_factor(rng, N, r_l)
    s = 2.0
    g1 = scalar_dev(2688.0)  # tensor scale g = 1
    layer = ft.prepare_layer(W_res=dev_bf16(Wr), U=dev_bf16(U), V=dev_bf16(V), A=dev_bf16(A), B=dev_bf16(B),
                             s=s, amax=g1)
    Xd, dYd = dev_bf16(X), dev_bf16(dY)
    Y, P = ft.ft_linear_fwd(layer, Xd, amax_x=g1, out_dtype=ft.F32)
    Yb, _ = ft.ft_linear_fwd(layer, Xd, amax_x=g1, out_dtype=ft.BF16)
    dX, dA, dB = ft.ft_linear_bwd(layer, dYd, Xd, P, amax_dy=g1, out_dtype=ft.F32)
    dXb, _, _ = ft.ft_linear_bwd(layer, dYd, Xd, P, amax_dy=g1, out_dtype=ft.BF16)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    f = oracle.bf16_to_f64
    Xf, dYf, Wf, Uf, Vf, Af, Bf = (f(t) for t in (X, dY, Wr, U, V, A, B))
    P_ref = np.concatenate([Xf @ Uf, s * (Xf @ Af)], axis=1)
    Pg_ref = np.concatenate([dYf @ Vf, s * (dYf @ Bf)], axis=1)
    for T in (P_ref, Pg_ref):
        assert np.array_equal(f(oracle.bf16_from_f64(T)), T)  # exact in bf16
    np.testing.assert_array_equal(host_u16(P), oracle.bf16_from_f64(P_ref))
    LRf = np.concatenate([Vf, Bf], axis=1)
    LRb = np.concatenate([Uf, Af], axis=1)
    refs = {
        "Y": (Xf @ Wf.T + P_ref @ LRf.T, np.abs(Xf) @ np.abs(Wf).T + np.abs(P_ref) @ np.abs(LRf).T),
        "dX": (dYf @ Wf + Pg_ref @ LRb.T, np.abs(dYf) @ np.abs(Wf) + np.abs(Pg_ref) @ np.abs(LRb).T),
        "dA": (Xf.T @ Pg_ref[:, r_s:], np.abs(Xf).T @ np.abs(Pg_ref[:, r_s:])),
        "dB": (dYf.T @ P_ref[:, r_s:], np.abs(dYf).T @ np.abs(P_ref[:, r_s:])),
    }
    got = {"Y": host(Y), "dX": host(dX), "dA": host(dA), "dB": host(dB)}
    for name, (ref, absdot) in refs.items():
        # the precondition of exactness: multiples of 2^-4 below 2^20
        assert absdot.max() < 2.0 ** 20 and np.array_equal(ref * 16, np.rint(ref * 16)), name
        assert np.abs(ref).max() > 0
        np.testing.assert_array_equal(got[name].astype(np.float64), ref, err_msg=name)
    np.testing.assert_array_equal(host_u16(Yb), oracle.bf16_from_f64(refs["Y"][0]))
    np.testing.assert_array_equal(host_u16(dXb), oracle.bf16_from_f64(refs["dX"][0]))


def test_tiny_workload_fwd_bwd():
    _run_and_compare(ft_synth.TINY, 0, bf16_check=True)


def test_attention_projection_full():
    _run_and_compare(ft_synth.ATTN, 1, bf16_check=True)


@pytest.mark.parametrize("wl", [2, 3])
def test_mlp_workloads_sampled_rows(wl):
    rows = np.sort(np.random.default_rng(100 + wl).choice(4608, 256, replace=False))
    _run_and_compare(ft_synth.WORKLOADS[wl], wl, rows=rows)


def test_dit_qkv_shape_sampled_rows():
    shape = ft_synth.dit_block_linears(0)[0]
    rows = np.sort(np.random.default_rng(7).choice(4608, 256, replace=False))
    _run_and_compare(shape, 4, rows=rows)


@pytest.mark.parametrize("M", [1, 37, 300, 1000])
def test_ragged_token_counts(M):
    _run_and_compare(ft_synth.TINY, 11, M=M)


@pytest.mark.parametrize("r_s,r_l", [(0, 0), (0, 32), (32, 0), (16, 112), (64, 64)])
def test_rank_variants(r_s, r_l):
    _run_and_compare(ft_synth.TINY, 12, M=256, r_s=r_s, r_l=r_l)


def test_zero_input_gives_zero_output():
    inp, U, V, Wr, layer = _prep(ft_synth.TINY, 13)
    X = torch.zeros(128, 256, dtype=torch.bfloat16, device="cuda")
    Y, P = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32)
    torch.cuda.synchronize()
    assert not Y.any() and not P.any()


def test_empty_batch_is_a_no_op():
    inp, U, V, Wr, layer = _prep(ft_synth.TINY, 14)
    X = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    Y, P = ft.ft_linear_fwd(layer, X)
    dX, dA, dB = ft.ft_linear_bwd(layer, torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda"), X, P)
    torch.cuda.synchronize()
    assert Y.shape == (0, 256) and dX.shape == (0, 256)
    assert not dA.any() and not dB.any()


@pytest.mark.parametrize("wl", [1, 2])
def test_repeated_runs_are_bitwise_identical(wl):
    """Every reduction (split down-projection, adapter gradients, amax) adds
    in a fixed order and every shared-memory stage is released only after
    all of its readers are done, so repeated forward/backward passes must
    agree bit for bit; a cross-CTA ordering race or a stage overwritten
    under a reader would show up here.  The attention shape runs the
    single-pass resident quantizer; the MLP up-projection's backward
    (dY [4608, 12288]) runs the streaming two-pass one."""
    inp, U, V, Wr, layer = _prep(ft_synth.WORKLOADS[wl], 21)
    X, dY = dev_bf16(inp["X"]), dev_bf16(inp["dY"])
    ref = None
    for _ in range(6 if wl == 1 else 4):
        Y, P = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32)
        dX, dA, dB = ft.ft_linear_bwd(layer, dY, X, P, out_dtype=ft.F32)
        torch.cuda.synchronize()
        outs = [t.clone() for t in (Y, P, dX, dA, dB)]
        if ref is None:
            ref = outs
        else:
            for a, b in zip(outs, ref):
                assert torch.equal(a, b)


def _ws_qact(ws, M, N, K, r_s, r_l, C):
    co, so, go = ft.ft_workspace_qact(M, N, K, r_s, r_l)
    raw = ws.buf
    assert raw.numel() >= ft.ft_workspace_bytes(M, N, K, r_s, r_l)
    codes = host(raw[co:co + M * C // 2]).reshape(M, C // 2)
    scales = host(raw[so:so + M * C // 16]).reshape(M, C // 16)
    g = host(raw[go:go + 4]).view(np.float32)[0]
    return codes, scales, g


@pytest.mark.parametrize("case", ["tiny", "attn", "ragged300", "packed16_112", "rank0", "amax_given",
                                  "streaming"])
def test_fused_quantizer_output_is_bit_exact(case):
    """The operand the 4-bit GEMM consumes, Q(X) after the forward and Q(dY)
    after the backward, read back from the workspace: codes, scales and the
    tensor scale equal the oracle's bit for bit (integer work).  Covers the
    single-pass resident path with its grid-wide amax (attention shape), the
    split reductions, a ragged token count, the packed-factor mode (a rank
    above 64), no low-rank branch, a caller-supplied amax, and the streaming
    two-pass path (the MLP up-projection's dY [4608, 12288] is too large to
    keep resident)."""
    shape, seed, M, r_s, r_l, amax = ft_synth.TINY, 50, None, None, None, None
    if case == "attn":
        shape, seed = ft_synth.ATTN, 51
    elif case == "streaming":
        shape, seed = ft_synth.WORKLOADS[2], 52
    elif case == "ragged300":
        M = 300
    elif case == "packed16_112":
        M, r_s, r_l = 256, 16, 112
    elif case == "rank0":
        M, r_s, r_l = 256, 0, 0
    elif case == "amax_given":
        amax = 7.25
    inp, U, V, Wr, layer = _prep(shape, seed, M, r_s, r_l)
    X, dY = inp["X"], inp["dY"]
    Mr = X.shape[0]
    ws = ft.Workspace()
    Y, P = ft.ft_linear_fwd(layer, dev_bf16(X), out_dtype=ft.F32, ws=ws,
                            amax_x=None if amax is None else scalar_dev(amax))
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    codes, scales, g = _ws_qact(ws, Mr, layer.N, layer.K, layer.r_s, layer.r_l, layer.K)
    rc, rs_, rg = oracle.quantize_1x16(X, amax)
    assert np.float32(g) == np.float32(rg)
    np.testing.assert_array_equal(scales, rs_)
    np.testing.assert_array_equal(codes, rc)
    ft.ft_linear_bwd(layer, dev_bf16(dY), dev_bf16(X), P, out_dtype=ft.F32, ws=ws,
                     amax_dy=None if amax is None else scalar_dev(amax))
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    codes, scales, g = _ws_qact(ws, Mr, layer.N, layer.K, layer.r_s, layer.r_l, layer.N)
    rc, rs_, rg = oracle.quantize_1x16(dY, amax)
    assert np.float32(g) == np.float32(rg)
    np.testing.assert_array_equal(scales, rs_)
    np.testing.assert_array_equal(codes, rc)


def test_foreign_sync_words_time_out_then_zeroing_recovers():
    """The workspace's synchronisation words are epoch-tagged: anything an
    earlier call left is valid, but a value no call writes (here all ones)
    must make the bounded device waits run out and report it through the
    error word -- not pass early and compute from a wrong tensor amax -- and
    zero-filling the workspace once must restore bit-identical results."""
    inp, U, V, Wr, layer = _prep(ft_synth.WORKLOADS[1], 22, M=512)
    X = dev_bf16(inp["X"])
    ws = ft.Workspace()
    ws.get(ft.ft_workspace_bytes(X.shape[0], layer.N, layer.K, layer.r_s, layer.r_l), X.device)
    Y0, P0 = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32, ws=ws)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    ws.buf[:256].fill_(0xFF)
    ft.ft_linear_fwd(layer, X, out_dtype=ft.F32, ws=ws)
    torch.cuda.synchronize()
    assert ft.ft_device_error() != 0
    ws.buf.zero_()
    Y1, P1 = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32, ws=ws)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    assert torch.equal(Y0, Y1) and torch.equal(P0, P1)


def test_cooperative_and_plain_quantizer_launches_agree():
    """The single-pass quantizer's grid barrier works under both launch
    modes: a plain launch (the default; its CTAs start as the previous
    kernel's CTAs retire) and a cooperative one.  Both compute the same
    bytes, so forward and backward outputs agree bit for bit."""
    inp, U, V, Wr, layer = _prep(ft_synth.ATTN, 23)
    X, dY = dev_bf16(inp["X"]), dev_bf16(inp["dY"])
    outs = []
    try:
        for coop in (False, True, False):
            ft.ft_set_cooperative_quantizer(coop)
            Y, P = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32)
            dX, dA, dB = ft.ft_linear_bwd(layer, dY, X, P, out_dtype=ft.F32)
            torch.cuda.synchronize()
            assert ft.ft_device_error() == 0
            outs.append([t.clone() for t in (Y, P, dX, dA, dB)])
    finally:
        ft.ft_set_cooperative_quantizer(False)
    for o in outs[1:]:
        for a, b in zip(o, outs[0]):
            assert torch.equal(a, b)


@pytest.mark.parametrize("wl", ["tiny", "attn"])
def test_1x16_weight_groups_fwd_bwd(wl):
    """The granularity ablation (FourTune page, section 4, "Impact of
    Quantization Granularity", Table 5): W_res quantized in 1x16 groups along
    K for the forward and, independently, W_res^T along N for dgrad.  The
    weight's codes and scales are bit-exact in both orientations; Y, dX, dA,
    dB within the same bound as the method's 16x16 layer."""
    shape, seed = (ft_synth.TINY, 61) if wl == "tiny" else (ft_synth.ATTN, 62)
    inp = ft_synth.make_inputs(shape, seed)
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    layer = ft.prepare_layer(W_res=dev_bf16(Wr), U=dev_bf16(U), V=dev_bf16(V), A=dev_bf16(inp["A"]),
                             B=dev_bf16(inp["B"]), s=inp["s"], weight_blk=ft.BLK_1x16)
    qk = oracle.quantize_1x16(Wr)
    qn = oracle.quantize_1x16_colwise(Wr)
    np.testing.assert_array_equal(host(layer.w_k.codes), qk[0])
    np.testing.assert_array_equal(host(layer.w_k.scales), qk[1])
    np.testing.assert_array_equal(host(layer.w_n.codes), qn[0])
    np.testing.assert_array_equal(host(layer.w_n.scales), qn[1])
    X, dY = dev_bf16(inp["X"]), dev_bf16(inp["dY"])
    Y, P = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32)
    dX, dA, dB = ft.ft_linear_bwd(layer, dY, X, P, out_dtype=ft.F32)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    M = inp["X"].shape[0]
    rows = np.arange(M) if wl == "tiny" else np.random.default_rng(5).choice(M, 256, replace=False)
    f = oracle.linear_fwd(inp["X"], Wr, U, V, inp["A"], inp["B"], inp["s"], rows=rows, qw=qk, weight_blk="1x16")
    b = oracle.linear_bwd(inp["dY"], inp["X"], Wr, U, V, inp["A"], inp["B"], inp["s"], f["P"], rows=rows, qw=qn,
                          weight_blk="1x16")
    assert oracle.rel_fro(host(Y)[rows], f["Y"]) <= TOL
    assert oracle.rel_fro(host(dX)[rows], b["dX"]) <= TOL
    assert oracle.rel_fro(host(dA), b["dA"]) <= TOL
    assert oracle.rel_fro(host(dB), b["dB"]) <= TOL


@pytest.mark.parametrize("precision", ["W4A16G4", "W4A4G16", "W4A16G16"])
@pytest.mark.parametrize("wl", ["tiny", "attn"])
def test_precision_variants(precision, wl):
    """The precision configurations of the FourTune page's ablation (section
    4, Table 4): the weight stays 4-bit; a 16-bit side's GEMM reads the bf16
    activation (forward) or output gradient (dgrad) with the weight's bf16
    image on tcgen05 kind::f16.  The images equal e2m1(code) x block scale
    bit for bit; Y, dX, dA, dB match the oracle's variant within 1e-3
    relative Frobenius error and every entry within its FP32 summation
    bound; the 4-bit side is bit-identical to the method's own call."""
    shape, seed = (ft_synth.TINY, 81) if wl == "tiny" else (ft_synth.ATTN, 82)
    inp = ft_synth.make_inputs(shape, seed)
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    args = dict(W_res=dev_bf16(Wr), U=dev_bf16(U), V=dev_bf16(V), A=dev_bf16(inp["A"]), B=dev_bf16(inp["B"]),
                s=inp["s"])
    layer = ft.prepare_layer(**args, precision=precision)
    base = ft.prepare_layer(**args)
    qw = oracle.quantize_16x16(Wr)
    Wimg = oracle.bf16_to_f64(oracle.bf16_from_f64(oracle.dequant_16x16(qw[0], qw[2], 1.0, shape.N, shape.K)))
    if layer.wd_k is not None:
        np.testing.assert_array_equal(host(layer.wd_k.float()).astype(np.float64), Wimg)
    if layer.wd_n is not None:
        np.testing.assert_array_equal(host(layer.wd_n.float()).astype(np.float64), Wimg.T)
    X, dY = dev_bf16(inp["X"]), dev_bf16(inp["dY"])
    Y, P = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32)
    dX, dA, dB = ft.ft_linear_bwd(layer, dY, X, P, out_dtype=ft.F32)
    Y4, P4 = ft.ft_linear_fwd(base, X, out_dtype=ft.F32)
    dX4, dA4, dB4 = ft.ft_linear_bwd(base, dY, X, P4, out_dtype=ft.F32)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    M = inp["X"].shape[0]
    rows = np.arange(M) if wl == "tiny" else np.sort(np.random.default_rng(6).choice(M, 256, replace=False))
    f = oracle.linear_fwd(inp["X"], Wr, U, V, inp["A"], inp["B"], inp["s"], rows=rows, qw=qw, precision=precision)
    b = oracle.linear_bwd(inp["dY"], inp["X"], Wr, U, V, inp["A"], inp["B"], inp["s"], f["P"], rows=rows, qw=qw,
                          precision=precision)
    for got, ref in ((host(Y)[rows], f["Y"]), (host(dX)[rows], b["dX"]), (host(dA), b["dA"]), (host(dB), b["dB"])):
        assert oracle.rel_fro(got, ref) <= TOL, oracle.rel_fro(got, ref)
    assert torch.equal(P, P4)
    if "A16" not in precision:
        assert torch.equal(Y, Y4)
    if "G16" not in precision:
        assert torch.equal(dX, dX4) and torch.equal(dA, dA4) and torch.equal(dB, dB4)
    # element-wise: the 16-bit GEMM accumulates bf16 x (e2m1 x scale) products
    # in FP32 and scales by g_w once
    d = oracle.bf16_to_f64
    gw = float(host(layer.w_k.tscale)[0])
    Wq = Wimg * gw
    if "A16" in precision:
        LRf = np.concatenate([d(V), d(inp["B"])], axis=1)
        Pd = d(host_u16(P))[rows]
        Xr = d(inp["X"])[rows]
        check_fp32_sum_bound(host(Y)[rows], Xr @ Wq.T + Pd @ LRf.T,
                             np.abs(Xr) @ np.abs(Wq).T + np.abs(Pd) @ np.abs(LRf).T, shape.K)


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_epilogue_amax_is_exact(out_dtype):
    """amax_y: the GEMM epilogue raises the word to max|Y| over Y as stored
    (the next quantizer's tensor amax); a larger value already there stays."""
    shape = ft_synth.LinearShape("amax", 300, 512, 768, 32, 32, outlier_channels=4, outlier_factor=20.0)
    inp, U, V, Wr, layer = _prep(shape, 81, None, None, None)
    X = dev_bf16(inp["X"])
    ot = ft.BF16 if out_dtype == "bf16" else ft.F32
    am = torch.zeros(1, dtype=torch.float32, device="cuda")
    Y, _ = ft.ft_linear_fwd(layer, X, out_dtype=ot, amax_y=am)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    assert am.item() == Y.abs().max().float().item()
    big = torch.full((1,), 1e30, dtype=torch.float32, device="cuda")
    ft.ft_linear_fwd(layer, X, out_dtype=ot, amax_y=big)
    torch.cuda.synchronize()
    assert big.item() == np.float32(1e30)
