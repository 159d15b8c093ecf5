"""Pins of the oracle's NVFP4 block quantizer (1x16 and 16x16).

Checked against: closed forms (the block holding the tensor amax lands on the
top of both grids; zero tensors and zero blocks), exact round trips of
lossless inputs with power-of-two scales, brute-force nearest-grid-point
checks with the exact (float64) quotient, the 16x16 transpose invariant of the
FourTune page (section 3.2: one scale grid serves W and W^T), and hand-built
byte layouts (nibble order).
"""
import numpy as np
import pytest

import ft_synth
import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _codes_to_nibbles(codes):
    lo = codes & 0xF
    hi = codes >> 4
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def _rand_bf16(rng, shape, scale=1.0):
    return ft_synth.to_bf16_bits(rng.standard_normal(shape) * scale)


def test_nibble_order_and_byte_layout():
    # amax supplied so that g = 2^-1 exactly: values are grid * 2^-1 * 448/448
    # With amax = 2688 * 0.5: g = 0.5; a block with max 3.0 has sf = 3/(6*0.5) = 1
    x = np.zeros((1, 16))
    x[0, 0] = 3.0    # q = 3/(1*0.5) = 6   -> code 7
    x[0, 1] = -0.25  # q = -0.5            -> code 9
    x[0, 2] = 1.0    # q = 2               -> code 4
    codes, scales, g = oracle.quantize_1x16(ft_synth.to_bf16_bits(x), amax=1344.0)
    assert g == 0.5
    assert scales[0, 0] == 0x38  # 1.0
    assert codes[0, 0] == 0x97   # element 0 low nibble, element 1 high nibble
    assert codes[0, 1] == 0x04


def test_amax_block_hits_top_of_both_grids():
    rng = np.random.default_rng(10)
    for trial in range(20):
        x = _rand_bf16(rng, (32, 64), scale=10.0 ** rng.uniform(-20, 20))
        xf = ft_synth.bf16_bits_to_f32(x)
        r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
        codes, scales, g = oracle.quantize_1x16(x)
        assert scales[r, c // 16] == 0x7E  # 448
        nib = _codes_to_nibbles(codes)[r, c]
        assert nib & 7 == 7                # |code| = 6
        assert (nib >> 3) == (1 if xf[r, c] < 0 else 0)
        cr, _, s16, g16 = oracle.quantize_16x16(x)
        assert g16 == g
        assert s16[r // 16, c // 16] == 0x7E
        assert _codes_to_nibbles(cr)[r, c] & 7 == 7


def test_tensor_scale_closed_form():
    x = ft_synth.to_bf16_bits(np.array([[-3.0] + [0.5] * 15]))
    _, _, g = oracle.quantize_1x16(x)
    assert g == np.float32(3.0) / np.float32(2688.0)
    zero = np.zeros((16, 32), np.uint16)
    codes, scales, g = oracle.quantize_1x16(zero)
    assert g == 1.0 and not codes.any() and not scales.any()


def test_zero_block_gives_zero_scale_and_plus_zero_codes():
    x = np.zeros((1, 32))
    x[0, 16:] = 1.0
    xb = ft_synth.to_bf16_bits(x)
    xb[0, 3] = 0x8000  # -0.0 inside the all-zero block
    codes, scales, _ = oracle.quantize_1x16(xb)
    assert scales[0, 0] == 0 and not codes[0, :8].any()
    # a negative zero inside a non-zero block keeps its sign bit
    xb[0, 17] = 0x8000
    codes, _, _ = oracle.quantize_1x16(xb)
    assert _codes_to_nibbles(codes)[0, 17] == 8


@pytest.mark.parametrize("blk", ["1x16", "16x16"])
def test_lossless_inputs_round_trip(blk):
    rng = np.random.default_rng(11)
    br = 1 if blk == "1x16" else 16
    x = ft_synth.lossless_fp4_operand(rng, 64, 128, br, exp_range=(-3, 3))
    amax = 2688.0 * 2.0 ** 0  # g = 1 exactly; block maxima 6*2^e give sf = 2^e
    if blk == "1x16":
        codes, scales, g = oracle.quantize_1x16(x, amax)
        deq = oracle.dequant_1x16(codes, scales, g, 64, 128)
    else:
        codes, _, scales, g = oracle.quantize_16x16(x, amax)
        deq = oracle.dequant_16x16(codes, scales, g, 64, 128)
    assert g == 1.0
    assert np.array_equal(deq, oracle.bf16_to_f64(x))


@pytest.mark.parametrize("blk", ["1x16", "16x16"])
def test_codes_are_nearest_grid_points(blk):
    """Brute force: given the block's scale, every element's code is a grid
    point nearest to the exact quotient x / (sd g) (clamped to the grid);
    exact ties must take the even code."""
    rng = np.random.default_rng(12)
    x = _rand_bf16(rng, (48, 96))
    xf = oracle.bf16_to_f64(x)
    xf_outl = xf.copy()
    if blk == "1x16":
        codes, scales, g = oracle.quantize_1x16(x)
        sd = np.repeat(np.vectorize(oracle.e4m3_value)(scales), 16, axis=1)
    else:
        codes, _, scales, g = oracle.quantize_16x16(x)
        sd = np.repeat(np.repeat(np.vectorize(oracle.e4m3_value)(scales), 16, axis=0), 16, axis=1)
    nib = _codes_to_nibbles(codes)
    mag = GRID[nib & 7]
    q = np.abs(xf_outl) / (sd * g)
    dist = np.abs(q[..., None] - GRID[None, None, :])
    best = dist.min(axis=-1)
    mine = np.abs(q - mag)
    # float32 rounding of the quotient may move a value by ~2^-23 relative
    assert np.all(mine <= best + 1e-6 * np.maximum(q, 1.0))
    # the sign bit follows the input sign
    assert np.array_equal(nib >> 3, (np.signbit(xf)).astype(np.uint8))


@pytest.mark.parametrize("blk", ["1x16", "16x16"])
def test_scale_is_rne_of_block_amax_over_six_g(blk):
    """sd approximates amax_block / (6 g) to E4M3 precision (relative 2^-4 in
    the normal range), i.e. the block max maps near the E2M1 top value 6."""
    rng = np.random.default_rng(13)
    x = _rand_bf16(rng, (64, 64))
    xf = np.abs(oracle.bf16_to_f64(x))
    if blk == "1x16":
        _, scales, g = oracle.quantize_1x16(x)
        amax_b = xf.reshape(64, 4, 16).max(axis=2)
    else:
        _, _, scales, g = oracle.quantize_16x16(x)
        amax_b = xf.reshape(4, 16, 4, 16).max(axis=(1, 3))
    sd = np.vectorize(oracle.e4m3_value)(scales)
    target = amax_b / (6.0 * g)
    ok = target >= 2.0 ** -6  # normal E4M3 range
    assert np.all(np.abs(sd[ok] - target[ok]) <= target[ok] * 2.0 ** -4 + 1e-12)


def test_16x16_transpose_invariant():
    """Section 3.2: with 16x16 blocks, quantizing W^T gives exactly the
    transposed codes and the transposed scale grid of W."""
    rng = np.random.default_rng(14)
    w = _rand_bf16(rng, (64, 96), 0.02)
    cr, cc, s, g = oracle.quantize_16x16(w)
    crT, ccT, sT, gT = oracle.quantize_16x16(np.ascontiguousarray(w.T))
    assert gT == g
    assert np.array_equal(sT, s.T)
    assert np.array_equal(crT, cc)
    assert np.array_equal(ccT, cr)
    assert np.array_equal(_codes_to_nibbles(cc), _codes_to_nibbles(cr).T)


def test_colwise_copy_is_rowwise_quantization_of_transpose_with_shared_scale():
    rng = np.random.default_rng(15)
    x = _rand_bf16(rng, (64, 48))
    _, _, g = oracle.quantize_1x16(x)
    cc, sc, gc = oracle.quantize_1x16_colwise(x)
    assert gc == g and cc.shape == (48, 32) and sc.shape == (48, 4)
    # the element (r, c) of x is element (c, r) of the column-wise copy: its
    # block is x[16*(r//16):16*(r//16)+16, c]
    xf = np.abs(oracle.bf16_to_f64(x))
    amax_col_blocks = xf.reshape(4, 16, 48).max(axis=1).T  # [48, 4]
    top = amax_col_blocks == xf.max()
    assert np.all(sc[top] == 0x7E)


def test_supplied_amax_equals_computed_amax():
    rng = np.random.default_rng(16)
    x = _rand_bf16(rng, (32, 64))
    a = oracle.amax_bf16(x)
    assert a == np.max(np.abs(ft_synth.bf16_bits_to_f32(x)))
    c1, s1, g1 = oracle.quantize_1x16(x)
    c2, s2, g2 = oracle.quantize_1x16(x, a)
    assert g1 == g2 and np.array_equal(c1, c2) and np.array_equal(s1, s2)
