#!/usr/bin/env python
"""Throughput of the W4A4G4 triple-branch linear (FourTune) on B200.

One step = the whole hot path over one batch: tensor amax + fused
quantize/down-projection of X, the FP4 forward GEMM with the fused low-rank
epilogue, tensor amax + fused quantize/down-projection of dY, the FP4 dgrad
GEMM, and the adapter gradients dA, dB (plus, with N > 1 GPUs, the data-
parallel all-reduce of dA, dB).  The once-per-layer SVD split and the 16x16
weight quantization are preparation and run before timing.

Workload: the attention projection of a FLUX-like DiT at 1024x1024,
X [4608, 3072] bf16 (4096 image + 512 text tokens) with 1% outlier channels,
W [3072, 3072], stabilizer rank 32, LoRA rank 16; synthetic seeded inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  value = FP4 GEMM FLOP of all ranks' steps
(2 GEMMs x 2 M N K each) / device time of the steps (max over ranks).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "W4A4G4 linear fwd+bwd TFLOPS vs NVFP4 peak; quantize GB/s vs HBM peak"
UNIT = "TFLOP/s"
FP4_OVER_BF16 = 4.0  # nominal dense NVFP4 / dense bf16 tensor rate on B200 (9 / 2.25 PFLOP/s)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--sample-rows", type=int, default=256,
                    help="token rows per oracle step (reference arm / cpu baseline)")
    ap.add_argument("--skip-cpu-baseline", action="store_true",
                    help="omit the oracle timing (for profiler runs)")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def workload():
    import ft_synth
    return ft_synth.ATTN


def fp4_flops_per_step(shape, M=None):
    M = shape.M if M is None else M
    return 2 * (2.0 * M * shape.N * shape.K)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------- oracle leg
def oracle_sample_step(shape, inp, prep, rows):
    """The triple-branch forward + backward of the CPU oracle on a sub-batch
    of token rows (tensor scales from the full tensors)."""
    import oracle
    U, V, Wr, qw, amax_x, amax_dy = prep
    X = np.ascontiguousarray(inp["X"][rows])
    dY = np.ascontiguousarray(inp["dY"][rows])
    f = oracle.linear_fwd(X, Wr, U, V, inp["A"], inp["B"], inp["s"], amax_x=amax_x, qw=qw)
    oracle.linear_bwd(dY, X, Wr, U, V, inp["A"], inp["B"], inp["s"], f["P"], amax_dy=amax_dy, qw=qw)


def oracle_prep(shape, inp):
    import oracle
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    qw = oracle.quantize_16x16(Wr)
    return U, V, Wr, qw, oracle.amax_bf16(inp["X"]), oracle.amax_bf16(inp["dY"])


def cpu_baseline(shape, inp, rows_per_step, seconds=12.0):
    """Times the oracle as it stands on the host cores over a bounded sample."""
    prep = oracle_prep(shape, inp)
    rng = np.random.default_rng(123)
    done_rows, t_total, steps = 0, 0.0, 0
    while t_total < seconds and steps < 64:
        rows = np.sort(rng.choice(shape.M, rows_per_step, replace=False))
        t0 = time.perf_counter()
        oracle_sample_step(shape, inp, prep, rows)
        t_total += time.perf_counter() - t0
        done_rows += rows_per_step
        steps += 1
    flops = fp4_flops_per_step(shape, done_rows)
    return {
        "value": flops / t_total / 1e12,
        "unit": UNIT,
        "cores": blas_threads(),
        "kind": "oracle",
        "sample": f"{steps} oracle steps of {rows_per_step} token rows each "
                  f"(fwd+bwd of the {shape.name} linear on a row sub-batch, tensor scales "
                  f"from the full tensors), {t_total:.1f} s of host time",
    }


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import ft_synth
    shape = workload()
    inp = ft_synth.make_inputs(shape, seed=1)
    prep = oracle_prep(shape, inp)
    rng = np.random.default_rng(7)
    R = args.sample_rows
    for _ in range(args.warmup):
        oracle_sample_step(shape, inp, prep, np.sort(rng.choice(shape.M, R, replace=False)))
    times = []
    for _ in range(args.steps):
        rows = np.sort(rng.choice(shape.M, R, replace=False))
        t0 = time.perf_counter()
        oracle_sample_step(shape, inp, prep, rows)
        times.append(time.perf_counter() - t0)
    t_step = sum(times) / len(times)
    value = fp4_flops_per_step(shape, R) / t_step / 1e12
    out = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_step * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{shape.name} M={shape.M} K={shape.K} N={shape.N} r_s={shape.r_s} "
                               f"r_l={shape.r_l}; oracle step = {R}-row sub-batch",
                   "global_batch": R, "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: fwd+bwd on {R} random token rows of {shape.name}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


# ------------------------------------------------------------- GPU leg
class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (read-only)
    in a background thread while the timed region runs."""

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.dev = device_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        p = self.nvml
        while not self._stop.is_set():
            try:
                sm = p.nvmlDeviceGetClockInfo(self.h, p.NVML_CLOCK_SM)
                reasons = p.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                power = p.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((sm, reasons, power))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self._t:
            self._t.join()
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        p = self.nvml
        names = {
            "gpu_idle": p.nvmlClocksEventReasonGpuIdle,
            "applications_clocks_setting": p.nvmlClocksEventReasonApplicationsClocksSetting,
            "sw_power_cap": p.nvmlClocksEventReasonSwPowerCap,
            "hw_slowdown": p.nvmlClocksEventReasonHwSlowdown,
            "sync_boost": p.nvmlClocksEventReasonSyncBoost,
            "sw_thermal_slowdown": p.nvmlClocksEventReasonSwThermalSlowdown,
            "hw_thermal_slowdown": p.nvmlClocksEventReasonHwThermalSlowdown,
            "hw_power_brake_slowdown": p.nvmlClocksEventReasonHwPowerBrakeSlowdown,
        }
        seen = set()
        for _, r, _ in self.samples:
            for n, bit in names.items():
                if r & bit:
                    seen.add(n)
        return {
            "sm_mhz": statistics.median(s[0] for s in self.samples),
            "sm_max_mhz": self.max_mhz,
            "reasons": sorted(seen),
            "power_w_max": max(s[2] for s in self.samples),
            "samples": len(self.samples),
        }


_COMMENT = re.compile(r"/\*.*?\*/|//[^\n]*", re.S)


def kernel_source_sha(name: str) -> str:
    """Hash of a kernel's source file and the device headers every kernel
    includes, comments and blank runs left out, so a recorded ncu figure
    lapses when any of their code changes (and not when only a comment
    does)."""
    h = hashlib.sha256()
    for part in (name, "ft_ptx.cuh", "ft_nvfp4.cuh"):
        with open(os.path.join(ROOT, "bit_quantized_lora_b200", "csrc", part)) as f:
            code = _COMMENT.sub("", f.read())
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, source: str):
    """DRAM bytes per launch from the committed ncu summary, when it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel]
        if e.get("source_sha") == kernel_source_sha(source):
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def run_ours(args):
    import torch

    import ft_synth
    import bit_quantized_lora_b200 as ft

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    shape = workload()
    M, N, K, r_s, r_l = shape.M, shape.N, shape.K, shape.r_s, shape.r_l

    # synthetic inputs (weak scaling): the weights are replicas (one seed for
    # every rank), every rank owns its own batch of tokens
    from bit_quantized_lora_b200 import dp
    wts = ft_synth.make_inputs(shape, seed=1)
    inp = ft_synth.make_inputs(shape, seed=dp.rank_seed(1, rank))

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(dev).view(torch.bfloat16)

    X, dY = to_dev(inp["X"]), to_dev(inp["dY"])
    W, A, B = to_dev(wts["W"]), to_dev(wts["A"]), to_dev(wts["B"])
    layer = ft.prepare_layer(W, r_s, A=A, B=B, s=wts["s"])  # untimed preparation
    ws = ft.Workspace()
    ws.get(ft.ft_workspace_bytes(M, N, K, r_s, r_l), dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    P = torch.empty(M, r_s + r_l, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    # dA, dB in one buffer: the step's only exchange is its sum over ranks
    ag = dp.AdapterGrads(K, N, r_l, dev)
    grads, dA, dB = ag.flat, ag.dA, ag.dB
    # L2 flush between steps: write a buffer larger than the 126 MB L2, then
    # read another one, so each step starts with a cold L2 that holds neither
    # the step's data nor dirty lines awaiting write-back
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    class _Flush:
        @staticmethod
        def zero_():
            flush_w.zero_()
            flush_r.sum()

    flush = _Flush()

    def step(Xs, dYs):
        ft.ft_linear_fwd(layer, Xs, Y=Y, P=P, ws=ws)
        ft.ft_linear_bwd(layer, dYs, Xs, P, dX=dX, dA=dA, dB=dB, ws=ws)
        ag.allreduce()

    def keep_host_ahead():
        # a short device-side sleep so the whole step is enqueued before the
        # GPU reaches it: the step's events then time device work only
        torch.cuda._sleep(2_000_000)

    for _ in range(args.warmup):
        flush.zero_()
        step(X, dY)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0, "device error during warm-up"

    # ---------------- timed region (kernel inputs resident in HBM); the
    # library's per-kernel events stay off here and are taken in a separate
    # pass below, so they add nothing between the step's launches
    sampler = ClockSampler(local).start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    evs = []
    for _ in range(args.steps):
        flush.zero_()
        keep_host_ahead()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step(X, dY)
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t_wall = time.perf_counter() - t_wall0
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    assert ft.ft_device_error() == 0, "device error during the timed region"

    # ---------------- per-kernel durations: the same steps again, each
    # library launch bracketed by CUDA events on its stream
    ft.timing.reset()
    ft.timing.enable(True)
    for _ in range(args.steps):
        flush.zero_()
        keep_host_ahead()
        step(X, dY)
    torch.cuda.synchronize()
    ft.timing.enable(False)
    kt = {k: ft.timing.read(k) for k in ["k_gemm_fp4", "k_qres", "k_qdown", "k_amax_bf16",
                                         "k_lora_grad", "k_pack_lt", "k_lora_grad_reduce"]}
    total_launches = ft.timing.read("*")[1]  # the same launches as the timed steps
    assert ft.ft_device_error() == 0, "device error during the per-kernel pass"
    ms_step = dp.max_over_ranks(sum(step_ms) / len(step_ms), dev)

    # ---------------- end to end through the API with host buffers
    Xh = torch.from_numpy(np.ascontiguousarray(inp["X"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    dYh = torch.from_numpy(np.ascontiguousarray(inp["dY"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    gh = torch.empty(grads.numel(), dtype=torch.float32).pin_memory()
    Xd2, dYd2 = torch.empty_like(X), torch.empty_like(dY)
    e2e_ms = []
    if dist is not None:
        dist.barrier()
    for i in range(args.warmup + args.steps):
        flush.zero_()
        keep_host_ahead()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        Xd2.copy_(Xh, non_blocking=True)
        dYd2.copy_(dYh, non_blocking=True)
        step(Xd2, dYd2)
        gh.copy_(grads, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    ms_e2e = dp.max_over_ranks(sum(e2e_ms) / len(e2e_ms), dev)

    flops = fp4_flops_per_step(shape)
    value = dp.job_rate(flops, world, ms_step) / 1e12
    hbm_gbs, bf16_tflops, peak_src = measured_peaks()
    fp4_peak = bf16_tflops * FP4_OVER_BF16

    gemm_ms, gemm_n = kt["k_gemm_fp4"]
    gemm_flops = 2.0 * M * N * K
    gemm_achieved = gemm_flops / (gemm_ms / gemm_n * 1e-3) / 1e12
    # the fused quantize + down-projection: the single-pass resident kernel
    # (tensor amax included) when the input fits the GPU's shared memory,
    # else the amax pass followed by the streaming kernel
    qd_kernel = "k_qres" if kt["k_qres"][1] > 0 else "k_qdown"
    qd_ms, qd_n = kt[qd_kernel]
    # per launch: read the [M, C] bf16 input and [C, r] factor, write codes,
    # scales and P (C = K in the forward, N in the backward; equal here)
    qd_bytes = M * K * (2 + 0.5 + 1 / 16) + K * (r_s + r_l) * 2 + M * (r_s + r_l) * 2
    qd_gbs = qd_bytes / (qd_ms / qd_n * 1e-3) / 1e9
    am_ms, am_n = kt["k_amax_bf16"]
    am_gbs = (M * K * 2) / (am_ms / am_n * 1e-3) / 1e9 if am_n else None
    lg_ms, lg_n = kt["k_lora_grad"]
    lg_gbs = (M * (N + K) * 2 + 2 * M * (r_s + r_l) * 2) / (lg_ms / lg_n * 1e-3) / 1e9

    out = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4",
        "data": "synthetic (seeded; FLUX-like DiT attention projection shapes, random-init weights)",
        "config": {
            "workload": f"{shape.name}: X [{M},{K}] bf16 (1% outlier channels x30), W [{N},{K}], "
                        f"stabilizer rank {r_s}, LoRA rank {r_l}; fwd + dgrad + LoRA grads",
            "global_batch": M * world,
            "seq_len": M,
            "parallelism": f"dp{world}" if world > 1 else "single",
            "l2": "flushed between steps (256 MB write then 256 MB read, outside the step events)",
        },
        "roofline": {
            "kernel": "k_gemm_fp4",
            "bound": "tensor",
            "achieved": gemm_achieved,
            "peak": fp4_peak,
            "unit": "TFLOP/s",
            "frac": gemm_achieved / fp4_peak,
            "traffic": ncu_traffic("k_gemm_fp4", "k_gemm_fp4.cuh"),
            "peak_source": f"{peak_src} bf16 {bf16_tflops} TFLOP/s x {FP4_OVER_BF16} (nominal NVFP4/bf16)",
            "flop_per_launch": gemm_flops,
            "launch_ms": gemm_ms / gemm_n,
        },
        "quantize": {
            "kernel": qd_kernel,
            "achieved": qd_gbs,
            "peak": hbm_gbs,
            "unit": "GB/s",
            "frac": qd_gbs / hbm_gbs,
            "bytes_per_launch": qd_bytes,
            "launch_ms": qd_ms / qd_n,
            "amax_gbs": am_gbs,
            "lora_grad_gbs": lg_gbs,
            "lora_grad_traffic": ncu_traffic("k_lora_grad", "k_lora_grad.cuh"),
            "traffic": ncu_traffic(qd_kernel, qd_kernel + ".cuh"),
        },
        "kernels_ms_per_step": {k: v[0] / args.steps for k, v in kt.items()},
        "gpu_launches": total_launches,
        "wall_s_timed_region": t_wall,
        "clocks": clocks,
        "e2e": {
            "value": dp.job_rate(flops, world, ms_e2e) / 1e12,
            "unit": UNIT,
            "h2d_bytes_per_step": X.numel() * 2 + dY.numel() * 2,
            "d2h_bytes_per_step": grads.numel() * 4,
        },
    }
    if world == 1 and rank == 0 and not args.skip_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(shape, inp, args.sample_rows)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
