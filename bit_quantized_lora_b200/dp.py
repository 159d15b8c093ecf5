"""Data parallelism for the triple-branch linear: one process per GPU, every
rank holding a replica of the frozen quantized backbone (Q(W_res), U, V) and
of the adapter (A, B), and running its own batch of tokens (FourTune page,
section 4: training on 8-GPU Blackwell platforms).

The backward's adapter gradients (FourTune page, section 3.2, Eq. 3) are
sums over token rows, dB = P_lora^T dY and dA = X^T Pg_lora, and each row of
P_lora = bf16(s X A) and Pg_lora = bf16(s dY B) depends on its own token row
only.  So the gradient of the whole job's batch is the sum over ranks of each
rank's gradient on its rows: one sum all-reduce of (dA, dB) per layer and
step is the only exchange.  Nothing else crosses ranks: each rank quantizes
its own activations and gradients with its own tensor scales, and Y, dX stay
on the rank that owns the rows.

The helpers below are the host side of that exchange and of the job's
timing (the slowest rank sets the step time); they run on any
torch.distributed backend (NCCL on GPUs, gloo on the CPU for tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: every rank draws its own tokens."""
    return base + rank


class AdapterGrads:
    """dA [K, r_l] and dB [N, r_l] (FP32, the library's output type, unless
    dtype says otherwise) as views of one flat buffer, so the
    per-step exchange is a single all-reduce; the library writes dA and dB
    in place (they are overwritten, not accumulated, by each backward)."""

    def __init__(self, K: int, N: int, r_l: int, device, dtype=torch.float32) -> None:
        self.flat = torch.empty(K * r_l + N * r_l, dtype=dtype, device=device)
        self.dA = self.flat[:K * r_l].view(K, r_l)
        self.dB = self.flat[K * r_l:].view(N, r_l)

    def allreduce(self, group=None, async_op: bool = False):
        """Sum over the ranks of the group, in place.  With async_op the
        exchange is only started and its handle returned: a training loop
        overlaps it with the next layer's backward and calls wait() before
        the optimizer reads dA, dB (None when there is nothing to exchange).

        An exchange in flight occupies SMs.  The library's single-pass
        quantizer (a layer call with no tensor amax supplied) joins its CTAs
        at a grid-wide barrier, so launched plainly beside a running
        all-reduce it can find some of its CTAs unscheduled: its bounded wait
        then gives up and ft_device_error() reports a timeout.  While
        exchanges overlap layer calls, either switch the quantizer to a
        cooperative launch (ft_set_cooperative_quantizer(True), as
        stack.LinearStack.step does), supply the tensor amax, or read
        ft_device_error() after the step.
        """
        if dist.is_initialized() and dist.get_world_size(group) > 1:
            return dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
        return None


def max_over_ranks(x: float, device=None, group=None) -> float:
    """The largest value of x over the ranks (the job's step time is the
    slowest rank's)."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: the units every rank processed in one step,
    divided by the slowest rank's step time (units per second)."""
    if max_ms <= 0:
        raise ValueError("step time must be positive")
    return world * units_per_rank / (max_ms * 1e-3)
