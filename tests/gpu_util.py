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
