"""GPU parity of the NVFP4 quantize kernels against the CPU oracle.

Codes, scales and the tensor scale must match bit for bit (integer work)."""
import numpy as np
import pytest
import torch

import ft_synth
import oracle
import bit_quantized_lora_b200 as ft
from gpu_util import dev_bf16, host, scalar_dev

pytestmark = pytest.mark.gpu


def _check_1x16(x_u16, amax=None):
    x = dev_bf16(x_u16)
    q = ft.ft_quantize(x, ft.BLK_1x16, amax=None if amax is None else scalar_dev(amax))
    torch.cuda.synchronize()
    codes, scales, g = oracle.quantize_1x16(x_u16, amax)
    assert np.float32(host(q.tscale)[0]) == np.float32(g)
    np.testing.assert_array_equal(host(q.scales), scales)
    np.testing.assert_array_equal(host(q.codes), codes)


@pytest.mark.parametrize("wl", [0, 1, 3])
def test_quantize_1x16_workload_activations_and_gradients(wl):
    shape = ft_synth.WORKLOADS[wl]
    inp = ft_synth.make_inputs(shape, seed=wl)
    _check_1x16(inp["X"])
    _check_1x16(inp["dY"])


def test_quantize_1x16_every_bf16_value():
    # all finite bf16 patterns, shuffled into 16-element blocks, under several
    # tensor scales (computed, larger, smaller than the true amax)
    rng = np.random.default_rng(30)
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = (bits.astype(np.uint32) << 16).view(np.float32)
    finite = bits[np.isfinite(f)]
    x = rng.permutation(finite)
    x = x[: (len(x) // 256) * 256].reshape(-1, 256)
    _check_1x16(x)
    for amax in [1.0, 3.0e38, 1e-30, 448.0 * 6.0]:
        _check_1x16(x, amax)
    # small-magnitude tensor: exercises subnormal divisors
    small = rng.permutation(finite[(np.abs(f[np.isfinite(f)]) < 1e-30)])
    small = small[: (len(small) // 256) * 256].reshape(-1, 256)
    _check_1x16(small)


def test_quantize_1x16_ragged_strided_zero():
    rng = np.random.default_rng(31)
    x = ft_synth.to_bf16_bits(rng.standard_normal((37, 80)))
    _check_1x16(x)
    # strided input (ld > cols): quantize a column slice
    big = ft_synth.to_bf16_bits(rng.standard_normal((40, 96)))
    xd = dev_bf16(big)[:, :64]
    q = ft.ft_quantize(xd, ft.BLK_1x16)
    torch.cuda.synchronize()
    codes, scales, g = oracle.quantize_1x16(np.ascontiguousarray(big[:, :64]))
    np.testing.assert_array_equal(host(q.codes), codes)
    np.testing.assert_array_equal(host(q.scales), scales)
    # all zero: g = 1, zero codes and scales
    z = np.zeros((16, 32), np.uint16)
    q = ft.ft_quantize(dev_bf16(z), ft.BLK_1x16)
    torch.cuda.synchronize()
    assert host(q.tscale)[0] == 1.0 and not host(q.codes).any() and not host(q.scales).any()


@pytest.mark.parametrize("wl", [0, 1, 2, 3])
def test_quantize_transpose_16x16_weights(wl):
    shape = ft_synth.WORKLOADS[wl]
    W = ft_synth.make_inputs(shape, seed=wl)["W"]
    cr, cc, s, g = oracle.quantize_16x16(W)
    w_k, w_n = ft.ft_quantize_transpose(dev_bf16(W), ft.BLK_16x16)
    torch.cuda.synchronize()
    assert np.float32(host(w_k.tscale)[0]) == np.float32(g)
    assert w_n.scales.data_ptr() == w_k.scales.data_ptr()
    np.testing.assert_array_equal(host(w_k.scales), s)
    np.testing.assert_array_equal(host(w_k.codes), cr)
    np.testing.assert_array_equal(host(w_n.codes), cc)
    # ft_quantize with 16x16 blocks emits the row layout alone, identically
    q = ft.ft_quantize(dev_bf16(W), ft.BLK_16x16)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(q.codes), cr)
    np.testing.assert_array_equal(host(q.scales), s)


@pytest.mark.parametrize("wl", [0, 2])
def test_quantize_transpose_1x16_activations(wl):
    shape = ft_synth.WORKLOADS[wl]
    inp = ft_synth.make_inputs(shape, seed=wl)
    for key in ["X", "dY"]:
        x = inp[key]
        r, c = ft.ft_quantize_transpose(dev_bf16(x), ft.BLK_1x16)
        torch.cuda.synchronize()
        cr, sr, g = oracle.quantize_1x16(x)
        cc, sc, gc = oracle.quantize_1x16_colwise(x)
        assert gc == g
        assert np.float32(host(r.tscale)[0]) == np.float32(g)
        assert np.float32(host(c.tscale)[0]) == np.float32(g)
        np.testing.assert_array_equal(host(r.codes), cr)
        np.testing.assert_array_equal(host(r.scales), sr)
        np.testing.assert_array_equal(host(c.codes), cc)
        np.testing.assert_array_equal(host(c.scales), sc)


@pytest.mark.parametrize("rows,cols,ld", [(16, 16, 16), (48, 144, 144), (80, 208, 216), (208, 400, 400),
                                          (96, 256, 264), (64, 128, 128)])
def test_quantize_transpose_ragged_tiles(rows, cols, ld):
    """Both layouts on shapes that leave partial 64 x 128 tiles (rows or
    columns not a multiple of the tile, row strides wider than the matrix):
    every partial store path -- byte scales, 8-byte column-code pieces --
    writes exactly the oracle's bytes and nothing past them (the outputs are
    pre-filled with a marker)."""
    rng = np.random.default_rng(rows * 1000 + cols)
    full = ft_synth.to_bf16_bits(rng.standard_normal((rows, ld)) * np.exp(rng.standard_normal((rows, ld))))
    xd = dev_bf16(full)[:, :cols]
    x = np.ascontiguousarray(full[:, :cols])
    for blk in (ft.BLK_16x16, ft.BLK_1x16):
        out_row = ft.FP4.empty(rows, cols, blk, "cuda")
        if blk == ft.BLK_16x16:
            out_col = ft.FP4.empty(cols, rows, blk, "cuda", scales=out_row.scales, tscale=out_row.tscale)
        else:
            out_col = ft.FP4.empty(cols, rows, blk, "cuda")
        for t in (out_row.codes, out_row.scales, out_col.codes, out_col.scales):
            t.fill_(0xA5)
        ft.ft_quantize_transpose(xd, blk, out_row=out_row, out_col=out_col)
        torch.cuda.synchronize()
        if blk == ft.BLK_16x16:
            cr, cc, sg, g = oracle.quantize_16x16(x)
            np.testing.assert_array_equal(host(out_row.codes), cr)
            np.testing.assert_array_equal(host(out_col.codes), cc)
            np.testing.assert_array_equal(host(out_row.scales), sg)
        else:
            cr, sr, g = oracle.quantize_1x16(x)
            cc, sc, _ = oracle.quantize_1x16_colwise(x)
            np.testing.assert_array_equal(host(out_row.codes), cr)
            np.testing.assert_array_equal(host(out_row.scales), sr)
            np.testing.assert_array_equal(host(out_col.codes), cc)
            np.testing.assert_array_equal(host(out_col.scales), sc)
            assert np.float32(host(out_col.tscale)[0]) == np.float32(g)
        assert np.float32(host(out_row.tscale)[0]) == np.float32(g)


def test_supplied_amax_matches_computed():
    rng = np.random.default_rng(32)
    x = ft_synth.to_bf16_bits(rng.standard_normal((64, 128)) * 3)
    a = oracle.amax_bf16(x)
    q1 = ft.ft_quantize(dev_bf16(x), ft.BLK_1x16)
    q2 = ft.ft_quantize(dev_bf16(x), ft.BLK_1x16, amax=scalar_dev(a))
    torch.cuda.synchronize()
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.scales, q2.scales)
    assert torch.equal(q1.tscale, q2.tscale)


def _boundary_probe(amax: float) -> np.ndarray:
    """bf16 tensor whose tensor amax is `amax` and whose 1x16 blocks, for
    every scale byte, hold the bf16 values next to each E2M1 rounding boundary
    (0.25, 0.75, ..., 5) times that byte's divisor: the inputs on which a
    quantizer that multiplies by a reciprocal instead of dividing would err."""
    g = np.float32(np.float32(amax) / np.float32(2688.0))
    bounds = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    rows = []
    for s in range(1, 0x7E):
        e, m = (s >> 3) & 0xF, s & 7
        sd = (m / 8.0) * 2.0**-6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        d = np.float32(np.float32(sd) * g)
        vals = []
        for bk in bounds:
            x0 = int(np.array([np.float32(bk) * d], dtype=np.float32).view(np.uint32)[0]) >> 16
            vals += [x0 - 1, x0, x0 + 1, x0 + 2]
        # the block max that selects this byte: 6 * sd * g, to bf16
        top = ft_synth.to_bf16_bits(np.array([6.0 * sd * float(g)]))[0]
        blk = np.array(vals[:15] + [top], dtype=np.uint32)
        blk2 = np.array(vals[15:] + [top] * (16 - len(vals[15:])), dtype=np.uint32)
        for b in (blk, blk2):
            b = np.clip(b, 0, 0x7F7F).astype(np.uint16)
            rows.append(b)
            rows.append(b | np.uint16(0x8000))  # the same magnitudes negative
    x = np.concatenate(rows)
    x = np.concatenate([x, ft_synth.to_bf16_bits(np.array([amax] * 16))])
    pad = (-len(x)) % 256
    x = np.concatenate([x, np.zeros(pad, dtype=np.uint16)])
    return x.reshape(-1, 256)


@pytest.mark.parametrize("amax", [5.40625, 1.0, 135.0, 0.0123, 7.3e-3, 2.2e4])
def test_quantize_1x16_rounding_boundaries_every_scale(amax):
    # 5.40625 is a tensor amax for which RN(1/d) misencodes one bf16 value for
    # every scale byte with mantissa 4: the quantizer must still match the
    # correctly rounded division bit for bit
    x = _boundary_probe(amax)
    a_bf16 = ft_synth.bf16_bits_to_f32(ft_synth.to_bf16_bits(np.array([amax])))[0]
    assert oracle.amax_bf16(x) == a_bf16
    _check_1x16(x)
    _check_1x16(x, float(oracle.amax_bf16(x)))
