"""Helpers shared by the GPU parity tests (numpy bf16 bit patterns <-> torch)."""
import numpy as np
import torch


def dev_bf16(u16: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(np.asarray(u16, np.uint16)).view(np.int16)
    return torch.from_numpy(a).cuda().view(torch.bfloat16)


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def scalar_dev(v: float) -> torch.Tensor:
    return torch.tensor([v], dtype=torch.float32, device="cuda")


def bf16_ulp_diff(a_u16: np.ndarray, b_u16: np.ndarray) -> np.ndarray:
    """|a - b| in units of bf16 ulps (sign-magnitude ordering)."""
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, -(u & 0x7FFF), u & 0x7FFF)
    return np.abs(key(a_u16) - key(b_u16))


def bf16_ulp_of(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (2^(e-7) for v in [2^e, 2^(e+1)))."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.ldexp(1.0, (e - 7).astype(int)), 2.0 ** -133)


def check_lowrank_down(P_gpu_u16, P_ref_u16, Td, L1d, L2d, s):
    """P = [bf16(T L1) | bf16(s T L2)] from an FP32 accumulation: each entry
    may differ from the FP64-accumulated reference by one bf16 rounding plus
    the FP32 summation error bound K 2^-23 sum_k |T_k L_k| (which dominates
    where the sum cancels)."""
    import oracle
    K = Td.shape[1]
    absT = np.abs(Td)
    mags = []
    if L1d.shape[1]:
        mags.append(absT @ np.abs(L1d))
    if L2d.shape[1]:
        mags.append(abs(s) * (absT @ np.abs(L2d)))
    mag = np.concatenate(mags, axis=1)
    got = oracle.bf16_to_f64(P_gpu_u16)
    ref = oracle.bf16_to_f64(P_ref_u16)
    bound = bf16_ulp_of(ref) + K * 2.0 ** -23 * mag + bf16_ulp_of(mag * K * 2.0 ** -23)
    excess = np.abs(got - ref) - bound
    assert np.all(excess <= 0), float(excess.max())


def check_fp32_sum_bound(got, ref, absdot, terms, slack=None):
    """Each entry of an FP32-accumulated result within the worst-case error
    of recursive FP32 summation of its `terms` products, terms * 2^-23 *
    sum |products| (absdot), plus one final FP32 rounding of the value
    (and `slack`, an allowance for operands that were themselves rounded
    differently, when given).  A single wrong entry -- a dropped or
    duplicated block, a stale tile -- breaks this bound even where a norm
    over the whole output would not notice it."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bound = terms * 2.0 ** -23 * np.asarray(absdot, np.float64) + 2.0 ** -23 * np.abs(ref) + 1e-30
    if slack is not None:
        bound = bound + slack
    excess = np.abs(got - ref) - bound
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert np.all(excess <= 0), (float(excess[worst]), worst, float(got[worst]), float(ref[worst]))


def lossless_operand(rng, rows, cols, block_rows, exp_range=(-1, 1)):
    """bf16 bits of a [rows, cols] matrix whose every block_rows x 16 block
    holds E2M1 grid values times one power of two, with a +-6 element in
    the block's first position, so that block quantization with tensor
    scale 1 is lossless (drawn in whole arrays: grid indices, signs, block
    exponents, first-element signs)."""
    import ft_synth
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    v = grid[rng.integers(0, 8, size=(rows, cols))] * rng.choice([-1.0, 1.0], size=(rows, cols))
    nb = (rows // block_rows, cols // 16)
    e = rng.integers(exp_range[0], exp_range[1] + 1, size=nb)
    v[::block_rows, ::16] = 6.0 * rng.choice([-1.0, 1.0], size=nb)
    v *= np.ldexp(1.0, np.repeat(np.repeat(e, block_rows, axis=0), 16, axis=1))
    return ft_synth.to_bf16_bits(v)


def selection_factor(rng, rows, r, exps=(-1, 0, 1)):
    """bf16 bits of a [rows, r] factor with exactly one nonzero, +-2^e, per
    column, in distinct rows: products with it are exact and its low-rank
    sums have a single term."""
    import ft_synth
    F = np.zeros((rows, r))
    idx = rng.choice(rows, r, replace=False)
    F[idx, np.arange(r)] = rng.choice([-1.0, 1.0], size=r) * np.ldexp(1.0, rng.choice(exps, size=r))
    return ft_synth.to_bf16_bits(F)
