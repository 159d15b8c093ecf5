"""A stack of triple-branch W4A4G4 linears run as one training step.

FourTune replaces every linear layer of a diffusion transformer with the
triple-branch layer (section 3.1) and reports the DiT training step as a
whole (section 4.2, efficiency).  `LinearStack` runs such a step over a list
of prepared layers on one stream: the forward (Eq. 2) of every layer in
order, then the backward (Eq. 3 and the adapter gradients) of every layer in
reverse order, each through the C ABI.  The attention and the activation
functions between the linears are not part of the method's path; every
layer here takes its own input X and output gradient dY.

One workspace serves every call: the calls are ordered on the stream, and
each kernel completes only after the kernels before it, so no call touches
the workspace while an earlier one still uses it.  The adapter gradients of
all layers are views of one flat FP32 buffer.  With data parallelism, each
layer's (dA, dB) all-reduce is started as soon as that layer's backward is
enqueued and overlaps the backward of the layers below it; the step waits
for every exchange at its end.  While exchanges run beside the backward,
the single-pass quantizer is launched cooperatively
(ft_set_cooperative_quantizer): its grid-wide barrier needs all of its CTAs
resident, which a plain launch cannot guarantee next to a collective kernel
on another stream that may hold SMs while it waits for a peer.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (BF16, Layer, Workspace, ft_linear_bwd, ft_linear_fwd, ft_set_cooperative_quantizer,
               ft_workspace_bytes)


@dataclass
class LayerBuffers:
    Y: torch.Tensor
    P: torch.Tensor
    dX: torch.Tensor
    dA: torch.Tensor | None
    dB: torch.Tensor | None


class LinearStack:
    """The layers of a stack and their output buffers for a batch of M
    tokens; outputs in `out_dtype` (bf16 by default, as a training step keeps
    them)."""

    def __init__(self, layers: list[Layer], M: int, device, out_dtype: int = BF16):
        self.layers = layers
        self.M = M
        self.out_dtype = out_dtype
        dt = torch.bfloat16 if out_dtype == BF16 else torch.float32
        n_grad = sum((L.K + L.N) * L.r_l for L in layers)
        self.grads = torch.zeros(max(n_grad, 1), dtype=torch.float32, device=device)
        self.bufs: list[LayerBuffers] = []
        self.grad_slices: list[torch.Tensor | None] = []
        off = 0
        for L in layers:
            dA = dB = sl = None
            if L.r_l > 0:
                n = (L.K + L.N) * L.r_l
                sl = self.grads[off:off + n]
                dA = sl[:L.K * L.r_l].view(L.K, L.r_l)
                dB = sl[L.K * L.r_l:].view(L.N, L.r_l)
                off += n
            self.bufs.append(LayerBuffers(
                Y=torch.empty(M, L.N, dtype=dt, device=device),
                P=torch.empty(M, L.r_s + L.r_l, dtype=torch.bfloat16, device=device),
                dX=torch.empty(M, L.K, dtype=dt, device=device), dA=dA, dB=dB))
            self.grad_slices.append(sl)
        self.ws = Workspace()
        self.ws.get(max(ft_workspace_bytes(M, L.N, L.K, L.r_s, L.r_l) for L in layers), device)

    def forward_layer(self, j: int, X: torch.Tensor, amax: torch.Tensor | None = None) -> None:
        b = self.bufs[j]
        ft_linear_fwd(self.layers[j], X, amax_x=amax, out_dtype=self.out_dtype, Y=b.Y, P=b.P, ws=self.ws)

    def backward_layer(self, j: int, dY: torch.Tensor, X: torch.Tensor, amax: torch.Tensor | None = None) -> None:
        b = self.bufs[j]
        ft_linear_bwd(self.layers[j], dY, X, b.P, amax_dy=amax, out_dtype=self.out_dtype, dX=b.dX, dA=b.dA,
                      dB=b.dB, ws=self.ws)

    def step(self, Xs: list[torch.Tensor], dYs: list[torch.Tensor], group=None, x_ready=None,
             dy_ready=None) -> None:
        """Forward of every layer in order, then backward in reverse order.
        With a process group of more than one rank, each layer's adapter
        gradients are summed over the ranks by an all-reduce started right
        after its backward; the step returns once the current stream has
        been made to wait for all of them.  x_ready / dy_ready: optional
        CUDA events, one per layer, that the layer's forward / backward
        waits for first (inputs arriving on another stream, e.g. host copies
        overlapped with the layers before)."""
        import torch.distributed as dist
        exchange = dist.is_initialized() and dist.get_world_size(group) > 1
        stream = torch.cuda.current_stream() if (x_ready is not None or dy_ready is not None) else None
        for j in range(len(self.layers)):
            if x_ready is not None:
                stream.wait_event(x_ready[j])
            self.forward_layer(j, Xs[j])
        handles = []
        if exchange:
            ft_set_cooperative_quantizer(True)
        try:
            for j in reversed(range(len(self.layers))):
                if dy_ready is not None:
                    stream.wait_event(dy_ready[j])
                self.backward_layer(j, dYs[j], Xs[j])
                if exchange and self.grad_slices[j] is not None:
                    handles.append(dist.all_reduce(self.grad_slices[j], op=dist.ReduceOp.SUM, group=group,
                                                   async_op=True))
        finally:
            if exchange:
                ft_set_cooperative_quantizer(False)
        for h in handles:
            h.wait()
