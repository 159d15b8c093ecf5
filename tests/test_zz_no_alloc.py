"""ft_linear_fwd_noalloc: the forward for callers that cannot give the
library a workspace (no device allocator on their side, or a host framework
that owns all device memory).  It must produce what ft_linear_fwd produces,
call after call, with its scratch inside the library.  This file is named to
run last so a stop-at-first-failure run has already covered everything else.
"""
import ctypes

import pytest
import torch

import ft_synth
import oracle
import bit_quantized_lora_b200 as ft
from bit_quantized_lora_b200 import _lib
from gpu_util import dev_bf16, host

pytestmark = pytest.mark.gpu

TOL = 1e-3
FT_OK, FT_ERR_WORKSPACE = 0, 6


def _layer(shape, seed):
    inp = ft_synth.make_inputs(shape, seed)
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    inp["split"] = (U, V, Wr)
    layer = ft.prepare_layer(W_res=dev_bf16(Wr), U=dev_bf16(U), V=dev_bf16(V), A=dev_bf16(inp["A"]),
                             B=dev_bf16(inp["B"]), s=inp["s"])
    return inp, layer


def _noalloc(L, layer, X):
    M, r = X.shape[0], layer.r_s + layer.r_l
    Y = torch.full((M, layer.N), float("nan"), dtype=torch.float32, device="cuda")
    P = torch.zeros(M, r, dtype=torch.bfloat16, device="cuda")
    view = layer.view()
    stream = torch.cuda.current_stream().cuda_stream
    st = L.ft_linear_fwd_noalloc(ctypes.byref(view), X.data_ptr(), M, None, Y.data_ptr(), ft.F32,
                                 P.data_ptr(), stream)
    assert st == FT_OK, L.ft_status_str(st)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0
    return Y, P


@pytest.mark.parametrize("wl", [0, 1])
def test_noalloc_forward_matches_workspace_forward_twice(wl):
    """Two calls in a row share the static scratch; between them a call of
    another shape leaves its own codes, scales and counters in it.  The same
    kernels run on the same inputs as ft_linear_fwd, whose reductions add in
    a fixed order, so Y and P must equal its results bit for bit; a scratch
    left stale or partly overwritten would change them.  Y is also checked
    against the FP64 oracle (relative Frobenius error 1e-3)."""
    L = _lib.load()
    shape = ft_synth.WORKLOADS[wl]
    inp, layer = _layer(shape, wl)
    other_inp, other = _layer(ft_synth.WORKLOADS[1 - wl], 5)
    X, X_other = dev_bf16(inp["X"]), dev_bf16(other_inp["X"])
    Y_ref, P_ref = ft.ft_linear_fwd(layer, X, out_dtype=ft.F32)
    torch.cuda.synchronize()
    Y1, P1 = _noalloc(L, layer, X)
    Yo, _ = _noalloc(L, other, X_other)
    Y2, P2 = _noalloc(L, layer, X)
    for Y, P in ((Y1, P1), (Y2, P2)):
        assert torch.equal(Y, Y_ref)
        assert torch.equal(P, P_ref)
    assert not torch.isnan(Yo).any()
    if wl == 0:
        U, V, Wr = inp["split"]
        f = oracle.linear_fwd(inp["X"], Wr, U, V, inp["A"], inp["B"], inp["s"])
        assert oracle.rel_fro(host(Y2), f["Y"]) <= TOL


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = _lib.load()
    cap = L.ft_linear_fwd_noalloc_max_bytes()
    assert cap == 32 << 20
    inp, layer = _layer(ft_synth.TINY, 0)
    view = layer.view()
    # a token count whose workspace exceeds the static scratch is refused
    # on the host, before anything is launched
    M = 1
    while L.ft_workspace_bytes(M, layer.N, layer.K, layer.r_s, layer.r_l) <= cap:
        M *= 2
    st = L.ft_linear_fwd_noalloc(ctypes.byref(view), 0x1000, M, None, 0x1000, ft.F32, 0x1000, None)
    assert st == FT_ERR_WORKSPACE
