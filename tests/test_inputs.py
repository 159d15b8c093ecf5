"""The synthetic input recipe (seeded, generated on the host): the
statistics each workload is declared with, checked on row shards small
enough for the CPU suite.  The generator holds none of the method's
arithmetic; it feeds the oracle and the GPU path alike."""
import numpy as np
import pytest

import ft_synth


def _f(u16):
    return ft_synth.bf16_bits_to_f32(u16).astype(np.float64)


def test_bf16_rounding_of_the_generator_is_nearest_even():
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 3.0e-40, 0.0, -0.0])
    got = ft_synth.bf16_bits_to_f32(ft_synth.to_bf16_bits(v))
    # ties to even: 1 + 2^-8 -> 1, 1 + 3 * 2^-8 -> 1 + 2^-6
    np.testing.assert_array_equal(got[:3], np.float32([1.0, 1.0 + 2.0 ** -6, -1.0]))
    assert got[3] != 0 and abs(got[3] - 3.0e-40) <= 2.0 ** -133  # subnormals kept
    assert np.signbit(got[5]) and not np.signbit(got[4])


def test_same_seed_same_tensors_other_seed_other_tokens():
    a = ft_synth.make_inputs(ft_synth.TINY, 3)
    b = ft_synth.make_inputs(ft_synth.TINY, 3)
    c = ft_synth.make_inputs(ft_synth.TINY, 4)
    for k in ("X", "W", "A", "B", "dY"):
        np.testing.assert_array_equal(a[k], b[k])
    assert not np.array_equal(a["X"], c["X"])


def test_outlier_channels_of_the_attention_projection_input():
    shape = ft_synth.ATTN
    inp = ft_synth.make_inputs(shape, 1, M=512)
    X = _f(inp["X"])
    col_std = X.std(axis=0)
    big = np.sort(np.argsort(col_std)[-shape.outlier_channels:])
    assert shape.outlier_channels == round(0.01 * shape.K)  # 1 % of the channels
    # the amplified columns stand apart by the declared factor
    assert col_std[big].min() > 10 * np.median(col_std)
    assert np.median(col_std[big]) == pytest.approx(shape.outlier_factor, rel=0.1)
    rest = np.delete(col_std, big)
    assert np.median(rest) == pytest.approx(1.0, rel=0.05)
    assert _f(inp["W"]).std() == pytest.approx(shape.w_std, rel=0.02)
    assert _f(inp["A"]).std() == pytest.approx(0.01, rel=0.05)
    assert _f(inp["dY"]).std() == pytest.approx(1.0, rel=0.02)


def test_down_projection_inputs_are_gelu_activations_and_heavy_tailed_gradients():
    shape = ft_synth.MLP_DOWN
    inp = ft_synth.make_inputs(shape, 3, M=128)
    X = _f(inp["X"])
    # GELU(z) >= its minimum (about -0.170); over z ~ N(0, 1) its mean is
    # E[z Phi(z)] = 1 / (2 sqrt(pi)) = 0.2821
    assert X.min() >= -0.1701
    assert X.mean() == pytest.approx(0.2821, abs=0.01)
    dY = _f(inp["dY"])
    # Student t with 3 degrees of freedom, scale 1e-3: median |t3| = 0.765; heavy tails
    assert np.median(np.abs(dY)) == pytest.approx(0.765e-3, rel=0.05)
    assert np.abs(dY).max() > 20 * np.median(np.abs(dY))
    assert _f(inp["W"]).std() == pytest.approx(0.01, rel=0.02)
