"""Pins of the oracle's MLP pieces (FourTune page, section 3.3, MLP Fusion):
the bf16 GELU against a 50-digit evaluation on every bf16 value, and the
fused MLP forward's special cases."""
import numpy as np

import ft_synth
import oracle


def test_gelu_bf16_every_value_against_high_precision():
    """All 65536 bf16 inputs: the table equals GELU evaluated with 50
    significant digits and rounded once to nearest even (mpmath), so the
    float64 erfc path never lands on the wrong side of a bf16 midpoint."""
    import mpmath
    mpmath.mp.dps = 50
    u = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = oracle.bf16_to_f64(u)
    got = oracle.gelu_bf16(u)
    finite = np.isfinite(x)
    for i in np.nonzero(finite)[0]:
        xm = mpmath.mpf(float(x[i]))
        h = xm * mpmath.erfc(-xm / mpmath.sqrt(2)) / 2
        # exact RNE to bf16 of the high-precision value: compare against the
        # two bf16 neighbours of the float64 result
        ref = oracle.bf16_to_f64(np.array([got[i]], np.uint16))[0]
        if h == 0:
            assert ref == 0.0, i
            continue
        lo, hi = _bf16_neighbours(ref)
        assert abs(h - ref) <= abs(h - lo) and abs(h - ref) <= abs(h - hi), (i, float(x[i]))
        if abs(h - ref) == abs(h - lo) or abs(h - ref) == abs(h - hi):
            # an exact tie: even mantissa
            assert got[i] % 2 == 0, i
    # non-finite inputs pass through
    assert np.array_equal(np.isnan(oracle.bf16_to_f64(got)), np.isnan(x))


def _bf16_neighbours(v: float):
    b = oracle.bf16_from_f64(np.array([v]))[0].astype(np.int32)
    s = np.array([b - 1, b + 1], dtype=np.int64) & 0xFFFF
    if v == 0:
        return -2.0 ** -133, 2.0 ** -133
    n = oracle.bf16_to_f64(s.astype(np.uint16))
    return float(min(n)), float(max(n))


def test_gelu_closed_forms():
    x = np.array([0.0, 1.0, -1.0, 8.0, -8.0, 1e4, -1e4], np.float64)
    h = oracle.bf16_to_f64(oracle.gelu_bf16(oracle.bf16_from_f64(x)))
    assert h[0] == 0.0
    # GELU(y) = y Phi(y): Phi(1) = 0.8413447..., Phi(-1) = 0.1586552...
    assert abs(h[1] - 0.8413447460685429) <= 2 ** -8 and abs(h[2] + 0.15865525393145707) <= 2 ** -10
    # far from zero: y itself for y >> 0, a vanishing negative value for y << 0
    assert h[3] == 8.0 and h[5] == oracle.bf16_to_f64(oracle.bf16_from_f64(np.array([1e4])))[0]
    assert -1e-12 < h[4] <= 0.0 and h[6] == 0.0


def _layer(rng, N, K, r_s, r_l, w_std):
    W = ft_synth.to_bf16_bits(rng.standard_normal((N, K)) * w_std)
    U, V, Wr = oracle.svd_split(W, r_s)
    A = ft_synth.to_bf16_bits(rng.standard_normal((K, r_l)) * 0.01)
    B = ft_synth.to_bf16_bits(rng.standard_normal((N, r_l)) * 0.01)
    return dict(W_res=Wr, U=U, V=V, A=A, B=B, s=1.0)


def test_mlp_reduces_to_linear_where_gelu_is_the_identity():
    """Where every FC1 output is large and positive, GELU(y) rounds to y, so
    H equals the FC1 output and the fused MLP's down layer equals the plain
    linear forward on it; with the supplied amax equal to max|H| the
    quantized H equals the computed-amax quantization."""
    rng = np.random.default_rng(3)
    M, K, N, D = 32, 64, 128, 64
    X = ft_synth.to_bf16_bits(np.abs(rng.standard_normal((M, K))) + 1.0)
    up = _layer(rng, N, K, 8, 8, 0.02)
    up["W_res"] = ft_synth.to_bf16_bits(np.abs(rng.standard_normal((N, K))) * 0.5 + 0.5)
    down = _layer(rng, D, N, 8, 8, 0.02)
    Y_up = oracle.bf16_from_f64(oracle.linear_fwd(X, up["W_res"], up["U"], up["V"], up["A"], up["B"], 1.0)["Y"])
    assert oracle.bf16_to_f64(Y_up).min() > 10.0
    amax_h = oracle.amax_bf16(Y_up)
    m = oracle.mlp_fwd(X, up, down, amax_h)
    np.testing.assert_array_equal(m["H"], Y_up)
    f = oracle.linear_fwd(Y_up, down["W_res"], down["U"], down["V"], down["A"], down["B"], 1.0)
    np.testing.assert_array_equal(m["Y"], f["Y"])
    for a, b in zip(m["qh"], oracle.quantize_1x16(Y_up)):
        np.testing.assert_array_equal(a, b)


def test_mlp_is_row_local_and_zero_input():
    """Given the tensor amaxes, each token row of the fused MLP depends on
    that row alone (so sampled rows are exact), and X = 0 gives H = 0."""
    rng = np.random.default_rng(4)
    M, K, N, D = 48, 64, 128, 64
    X = ft_synth.to_bf16_bits(rng.standard_normal((M, K)))
    up, down = _layer(rng, N, K, 8, 8, 0.05), _layer(rng, D, N, 8, 8, 0.05)
    ax = oracle.amax_bf16(X)
    full = oracle.mlp_fwd(X, up, down, 3.0, amax_x=ax)
    rows = np.array([5, 17, 40])
    part = oracle.mlp_fwd(np.ascontiguousarray(X[rows]), up, down, 3.0, amax_x=ax)
    np.testing.assert_array_equal(part["H"], full["H"][rows])
    # (float64 products of a 3-row and a 48-row batch may sum in different orders)
    np.testing.assert_allclose(part["Y"], full["Y"][rows], rtol=1e-12, atol=1e-15)
    z = oracle.mlp_fwd(np.zeros((4, K), np.uint16), up, down, 3.0)
    assert not oracle.bf16_to_f64(z["H"]).any()
