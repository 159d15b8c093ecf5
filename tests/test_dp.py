"""The data-parallel path on the CPU: two gloo ranks (world size 2), each
with its own batch of tokens and the same replicated weights, exchange the
adapter gradients with the helpers bench.py uses over NCCL.

Pins: the all-reduced dA, dB equal the oracle's gradients on the two batches
stacked into one (FourTune page, section 3.2, Eq. 3: the adapter gradients
are sums over token rows, and P_lora, Pg_lora are row-wise); the job's step
time is the slowest rank's; the job rate counts every rank's work.  A rank
that leaves before the exchange makes the other rank's collective fail
within the process group's timeout instead of hanging."""
import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

WORLD = 2
BASE_SEED = 7


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank: int, port: int, timeout_s: float):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def _batch(rank: int):
    """Replicated weights (one seed for every rank) and this rank's tokens."""
    import ft_synth
    from bit_quantized_lora_b200 import dp
    shape = ft_synth.TINY
    w = ft_synth.make_inputs(shape, BASE_SEED)
    mine = ft_synth.make_inputs(shape, dp.rank_seed(BASE_SEED + 100, rank))
    return shape, w, mine["X"], mine["dY"]


def _oracle_grads(shape, w, X, dY):
    import oracle
    U, V, Wr = oracle.svd_split(w["W"], shape.r_s)
    qw = oracle.quantize_16x16(Wr)
    f = oracle.linear_fwd(X, Wr, U, V, w["A"], w["B"], w["s"], rows=np.arange(1), qw=qw)
    b = oracle.linear_bwd(dY, X, Wr, U, V, w["A"], w["B"], w["s"], f["P"], rows=np.arange(1), qw=qw)
    return b["dA"], b["dB"]


def _exchange_worker(rank: int, port: int, out: str):
    dist = _init(rank, port, 60.0)
    try:
        from bit_quantized_lora_b200 import dp
        shape, w, X, dY = _batch(rank)
        dA, dB = _oracle_grads(shape, w, X, dY)
        g = dp.AdapterGrads(shape.K, shape.N, shape.r_l, "cpu", dtype=torch.float64)
        g.dA.copy_(torch.from_numpy(dA))
        g.dB.copy_(torch.from_numpy(dB))
        g.allreduce()
        # the slowest rank sets the step time; the rate counts both ranks
        slow = dp.max_over_ranks(1.0 + rank)
        rate = dp.job_rate(10.0, WORLD, slow)
        np.savez(os.path.join(out, f"rank{rank}.npz"), dA=g.dA.numpy(), dB=g.dB.numpy(),
                 slow=slow, rate=rate)
    finally:
        dist.destroy_process_group()


def test_adapter_gradients_all_reduced_over_two_ranks_equal_the_full_batch():
    with tempfile.TemporaryDirectory() as out:
        mp.start_processes(_exchange_worker, args=(_free_port(), out), nprocs=WORLD, start_method="spawn")
        r = [np.load(os.path.join(out, f"rank{k}.npz")) for k in range(WORLD)]
    # every rank holds the same sum
    np.testing.assert_array_equal(r[0]["dA"], r[1]["dA"])
    np.testing.assert_array_equal(r[0]["dB"], r[1]["dB"])
    # ... which is the gradient of the stacked batch (rows of both ranks)
    shape, w, X0, dY0 = _batch(0)
    _, _, X1, dY1 = _batch(1)
    dA, dB = _oracle_grads(shape, w, np.concatenate([X0, X1]), np.concatenate([dY0, dY1]))
    for got, ref in ((r[0]["dA"], dA), (r[0]["dB"], dB)):
        assert np.abs(ref).max() > 0
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # the job's step time is the slowest rank's, and the rate counts both
    assert float(r[0]["slow"]) == float(r[1]["slow"]) == 2.0
    assert float(r[0]["rate"]) == pytest.approx(WORLD * 10.0 / 2e-3)


def _overlap_worker(rank: int, port: int, out: str):
    dist = _init(rank, port, 60.0)
    try:
        from bit_quantized_lora_b200 import dp
        # two layers' gradients: layer 1's exchange runs while layer 0's
        # gradients are computed, then both are awaited
        g1 = dp.AdapterGrads(8, 4, 16, "cpu", dtype=torch.float64)
        g0 = dp.AdapterGrads(8, 4, 16, "cpu", dtype=torch.float64)
        g1.flat.copy_(torch.arange(g1.flat.numel(), dtype=torch.float64) * (rank + 1))
        h = g1.allreduce(async_op=True)
        g0.flat.fill_(10.0 * (rank + 1))  # the next layer's backward
        h0 = g0.allreduce(async_op=True)
        h.wait()
        h0.wait()
        np.savez(os.path.join(out, f"ov{rank}.npz"), g1=g1.flat.numpy(), g0=g0.flat.numpy())
    finally:
        dist.destroy_process_group()


def test_asynchronous_exchange_overlaps_and_sums():
    with tempfile.TemporaryDirectory() as out:
        mp.start_processes(_overlap_worker, args=(_free_port(), out), nprocs=WORLD, start_method="spawn")
        r = [np.load(os.path.join(out, f"ov{k}.npz")) for k in range(WORLD)]
    n = r[0]["g1"].size
    for k in range(WORLD):
        np.testing.assert_array_equal(r[k]["g1"], np.arange(n, dtype=np.float64) * 3.0)
        np.testing.assert_array_equal(r[k]["g0"], np.full(n, 30.0))


def test_job_rate_rejects_a_nonpositive_time():
    from bit_quantized_lora_b200 import dp
    with pytest.raises(ValueError):
        dp.job_rate(1.0, 2, 0.0)


def _leaver_worker(rank: int, port: int, out: str):
    dist = _init(rank, port, 5.0)
    from bit_quantized_lora_b200 import dp
    g = dp.AdapterGrads(4, 4, 16, "cpu")
    g.flat.fill_(1.0)
    if rank == 1:
        # leaves between steps: no collective of its own is in flight
        return
    try:
        g.allreduce()
        result = "completed"
    except Exception as e:  # the exchange must fail, not hang
        result = "failed: " + type(e).__name__
    with open(os.path.join(out, "rank0.txt"), "w") as f:
        f.write(result)


def test_a_rank_that_leaves_makes_the_exchange_fail_not_hang():
    import time
    with tempfile.TemporaryDirectory() as out:
        t0 = time.monotonic()
        try:
            mp.start_processes(_leaver_worker, args=(_free_port(), out), nprocs=WORLD, start_method="spawn")
        except Exception:
            pass  # the leaver's exit may be reported by the launcher; rank 0's record decides
        elapsed = time.monotonic() - t0
        with open(os.path.join(out, "rank0.txt")) as f:
            result = f.read()
    assert result.startswith("failed"), result
    assert elapsed < 120.0


class _FakeLayer:
    """The fields of a prepared layer the stack driver reads (N, K, ranks);
    the layer's weights ride along for the stand-in backward."""

    def __init__(self, shape, w):
        self.N, self.K, self.r_s, self.r_l, self.s = shape.N, shape.K, shape.r_s, shape.r_l, w["s"]
        self.shape, self.w = shape, w


def _stack_worker(rank: int, port: int, out: str):
    """The stack driver's step over two layers with the library calls
    replaced by CPU stand-ins (the oracle's backward writes dA, dB): records
    the call order and the quantizer launch mode each backward saw, and the
    all-reduced per-layer gradients."""
    dist = _init(rank, port, 60.0)
    try:
        import ft_synth
        from bit_quantized_lora_b200 import dp, stack
        log, coop = [], [False]

        def to_t(u16):
            return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)

        def fake_fwd(L, X, amax_x=None, out_dtype=0, Y=None, P=None, ws=None):
            log.append(("fwd", L.tag))

        def fake_bwd(L, dY, X, P, amax_dy=None, out_dtype=0, dX=None, dA=None, dB=None, ws=None):
            log.append(("bwd", L.tag, coop[0]))
            Xn = X.view(torch.int16).numpy().view(np.uint16)
            dYn = dY.view(torch.int16).numpy().view(np.uint16)
            gA, gB = _oracle_grads(L.shape, L.w, Xn, dYn)
            dA.copy_(torch.from_numpy(gA).float())
            dB.copy_(torch.from_numpy(gB).float())

        stack.ft_linear_fwd, stack.ft_linear_bwd = fake_fwd, fake_bwd
        stack.ft_set_cooperative_quantizer = lambda on: coop.__setitem__(0, bool(on))
        layers, Xs, dYs = [], [], []
        for j in range(2):
            shape = ft_synth.TINY
            w = ft_synth.make_inputs(shape, BASE_SEED + 10 * j)
            mine = ft_synth.make_inputs(shape, dp.rank_seed(BASE_SEED + 100 + 10 * j, rank))
            L = _FakeLayer(shape, w)
            L.tag = j
            layers.append(L)
            Xs.append(to_t(mine["X"]))
            dYs.append(to_t(mine["dY"]))
        st = stack.LinearStack(layers, ft_synth.TINY.M, "cpu")
        st.step(Xs, dYs)
        np.savez(os.path.join(out, f"st{rank}.npz"), grads=st.grads.numpy(),
                 log=np.array([str(x) for x in log]), coop_after=coop[0])
    finally:
        dist.destroy_process_group()


def test_stack_step_exchanges_every_layer_during_the_backward():
    """Two ranks run the stack driver's step over two layers: forwards in
    order, backwards in reverse order, each backward with the cooperative
    quantizer launch on (the exchanges of earlier layers run beside it) and
    the plain launch restored after the step; every layer's all-reduced
    (dA, dB) slice equals the oracle's gradient of the two ranks' batches
    stacked into one (FourTune page, section 3.2: sums over token rows)."""
    import ft_synth
    from bit_quantized_lora_b200 import dp
    with tempfile.TemporaryDirectory() as out:
        mp.start_processes(_stack_worker, args=(_free_port(), out), nprocs=WORLD, start_method="spawn")
        r = [np.load(os.path.join(out, f"st{k}.npz")) for k in range(WORLD)]
    np.testing.assert_array_equal(r[0]["grads"], r[1]["grads"])
    assert list(r[0]["log"]) == [str(("fwd", 0)), str(("fwd", 1)), str(("bwd", 1, True)), str(("bwd", 0, True))]
    assert not bool(r[0]["coop_after"])
    shape = ft_synth.TINY
    off = 0
    for j in range(2):
        w = ft_synth.make_inputs(shape, BASE_SEED + 10 * j)
        b = [ft_synth.make_inputs(shape, dp.rank_seed(BASE_SEED + 100 + 10 * j, k)) for k in range(WORLD)]
        dA, dB = _oracle_grads(shape, w, np.concatenate([x["X"] for x in b]), np.concatenate([x["dY"] for x in b]))
        n = (shape.K + shape.N) * shape.r_l
        got = r[0]["grads"][off:off + n].astype(np.float64)
        ref = np.concatenate([dA.ravel(), dB.ravel()])
        # each rank's FP32 gradient, summed in FP32 by the exchange
        np.testing.assert_allclose(got, ref, rtol=0, atol=4 * 2.0 ** -24 * np.abs(ref).max() + 1e-12)
        off += n
