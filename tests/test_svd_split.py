"""The library's own SVD split (the once-per-layer preparation of Eq. 1,
`bit_quantized_lora_b200.svd_split`, torch float64 on the host) against the
oracle's split and against what the decomposition fixes.

Singular vectors are defined up to sign, so U and V are compared with the
oracle's after aligning each column's sign; W_res is checked as the single
round-to-nearest-even rounding of W - V U^T from the library's own rounded
factors.  Runs on the CPU."""
import numpy as np
import pytest
import torch

import ft_synth
import oracle
import bit_quantized_lora_b200 as ft
from gpu_util import bf16_ulp_diff


def _t(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("N,K,r", [(256, 256, 16), (512, 256, 32), (256, 768, 16), (384, 128, 0)])
def test_library_split_matches_oracle_split(N, K, r):
    """The factors equal the oracle's up to each singular vector's sign (bit
    for bit but for rare one-ulp differences: the two sides' float64
    products sum in different orders), and W_res is exactly the single RNE
    rounding of W - V U^T formed from the library's own rounded factors."""
    rng = np.random.default_rng(N + K + r)
    sig = rng.standard_normal((N, 8)) @ rng.standard_normal((8, K)) * 0.05
    W = ft_synth.to_bf16_bits(sig + rng.standard_normal((N, K)) * 0.02)
    U, V, Wr = ft.svd_split(_t(W), r)
    assert Wr.dtype == torch.bfloat16 and Wr.shape == (N, K)
    if r == 0:
        assert U is None and V is None
        np.testing.assert_array_equal(_u16(Wr), W)
        return
    Uo, Vo, Wro = oracle.svd_split(W, r)
    Uu, Vu = _u16(U), _u16(V)
    assert U.shape == (K, r) and V.shape == (N, r)
    # align each column's sign with the oracle's (flip = bf16 sign bit)
    flip = np.sign(oracle.bf16_to_f64(Uu) * oracle.bf16_to_f64(Uo)).sum(axis=0) < 0
    Uu = np.where(flip, Uu ^ 0x8000, Uu).astype(np.uint16)
    Vu = np.where(flip, Vu ^ 0x8000, Vu).astype(np.uint16)
    for a, b in ((Uu, Uo), (Vu, Vo)):
        d = bf16_ulp_diff(a, b)
        assert d.max() <= 1 and (d > 0).mean() < 1e-3
    Wd = oracle.bf16_to_f64(W)
    expect = oracle.bf16_from_f64(Wd - oracle.bf16_to_f64(_u16(V)) @ oracle.bf16_to_f64(_u16(U)).T)
    np.testing.assert_array_equal(_u16(Wr), expect)


def test_single_rounding_of_the_split():
    """float64 -> bf16 in the split rounds once, to nearest even, including
    just above a tie, where rounding through float32 first would fall back
    onto the tie and round to even instead."""
    from bit_quantized_lora_b200 import _bf16_rne
    x = torch.tensor([1 + 2 ** -8 + 2 ** -30, 1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8 + 2 ** -40),
                      3e-39, 0.0], dtype=torch.float64)
    got = _u16(_bf16_rne(x))
    np.testing.assert_array_equal(got, oracle.bf16_from_f64(x.numpy()))
    assert got[0] == 0x3F81 and got[1] == 0x3F80 and got[2] == 0x3F82


def test_library_split_is_the_best_rank_r_part():
    """U has orthonormal columns (to bf16 rounding) spanning the top-r right
    singular subspace, V = W U, and W_res + V U^T reconstructs W to the
    bf16 rounding of W_res (the oracle split is pinned the same way)."""
    rng = np.random.default_rng(3)
    N, K, r = 320, 256, 16
    W = ft_synth.to_bf16_bits(rng.standard_normal((N, K)) * 0.02
                              + rng.standard_normal((N, 4)) @ rng.standard_normal((4, K)) * 0.1)
    U, V, Wr = ft.svd_split(_t(W), r)
    Wd = oracle.bf16_to_f64(W)
    Ud, Vd, Wrd = (oracle.bf16_to_f64(_u16(x)) for x in (U, V, Wr))
    assert np.abs(Ud.T @ Ud - np.eye(r)).max() < 2e-2
    np.testing.assert_allclose(Vd, Wd @ Ud, rtol=0, atol=np.abs(Wd @ Ud).max() * 2 ** -7)
    rec = Wrd + Vd @ Ud.T
    assert np.abs(rec - Wd).max() <= np.abs(Wd).max() * 2 ** -8
    # the top-r right singular subspace: projecting it onto span(U) keeps it
    _, sv, vt = np.linalg.svd(Wd)
    P = Ud @ np.linalg.pinv(Ud)
    assert np.linalg.norm(P @ vt[:r].T - vt[:r].T) <= 0.05 * np.sqrt(r)
    # and the residual's top singular value is the (r+1)-th of W
    assert abs(np.linalg.svd(Wrd, compute_uv=False)[0] - sv[r]) <= 0.02 * sv[0]
