#!/usr/bin/env python
"""Throughput of the W4A4G4 triple-branch linear (FourTune) on B200.

Default workload (dit8): a random-init stack of 8 DiT blocks at hidden 3072,
24 heads, MLP 12288, batch 1 x 4608 tokens (4096 image + 512 text tokens of a
1024x1024 image); each block has four triple-branch linears -- QKV [9216,
3072], attention out [3072, 3072], MLP up [12288, 3072] and MLP down [3072,
12288] -- with stabilizer rank 32 and LoRA rank 32.  One step = the forward
(Eq. 2) of all 32 linears in order, then their backward (Eq. 3 and the
adapter gradients) in reverse order, each through the C ABI: per call the
tensor amax and fused quantize/down-projection of the input, the FP4 GEMM
with the fused low-rank epilogue, and in the backward the adapter
gradients; with N > 1 GPUs each layer's dA, dB all-reduce overlaps the
backward of the layers below it.  The once-per-layer SVD split and the 16x16
weight quantization are preparation and run before timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload dit8|attn_proj]

Prints one JSON line (rank 0).  value = FP4 GEMM FLOP of all ranks' steps
(2 GEMMs x 2 M N K per linear) / device time of the steps (max over ranks).
The same line carries the attention projection alone (a single linear) and
the standalone quantize kernels as secondary figures.
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
N_BLOCKS = 8
SEED = 100  # linear type j of the stack draws its tensors from seed SEED + j (weights) / rank_seed(.., rank)
KERNELS = ["k_gemm_fp4", "k_qres", "k_qdown", "k_amax_bf16", "k_lora_grad", "k_pack_lt", "k_quant_1x16",
           "k_quant_tile16", "k_gelu_bf16"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["dit8", "attn_proj"], default="dit8")
    ap.add_argument("--sample-rows", type=int, default=256,
                    help="token rows per linear per oracle step (reference arm / cpu baseline)")
    ap.add_argument("--skip-cpu-baseline", action="store_true",
                    help="omit the oracle timing (for profiler runs)")
    ap.add_argument("--single", choices=["qkv", "out", "up", "down", "mlp"], default=None,
                    help="profiling: prepare one DiT-stack linear and run its forward and backward --steps "
                         "times (prints 'ok', no timing)")
    ap.add_argument("--skip-extras", action="store_true",
                    help="omit the secondary figures (attention projection, standalone quantizers) "
                         "and the end-to-end leg (for profiler runs)")
    ap.add_argument("--gemm-mode", choices=["pairs", "single"], default="pairs",
                    help="tiling of the 4-bit GEMMs: CTA pairs on 256 x 256 tiles (default) or one CTA per "
                         "128 x 256 tile (same results)")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)) or None, \
            "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, None, "fallback"


def stack_shapes():
    """The four linear types of a block (the 8 blocks have the same shapes)."""
    import ft_synth
    return ft_synth.dit_block_linears(0)


def gemm_flops(shape, M=None):
    """FP4 GEMM FLOP of one forward + dgrad of a linear (2 GEMMs x 2 M N K)."""
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
def oracle_prep(shape, inp):
    import oracle
    U, V, Wr = oracle.svd_split(inp["W"], shape.r_s)
    qw = oracle.quantize_16x16(Wr)
    return U, V, Wr, qw, oracle.amax_bf16(inp["X"]), oracle.amax_bf16(inp["dY"])


def oracle_sample_step(inp, prep, rows):
    """The triple-branch forward + backward of the CPU oracle on a sub-batch
    of token rows (tensor scales from the full tensors)."""
    import oracle
    U, V, Wr, qw, amax_x, amax_dy = prep
    X = np.ascontiguousarray(inp["X"][rows])
    dY = np.ascontiguousarray(inp["dY"][rows])
    f = oracle.linear_fwd(X, Wr, U, V, inp["A"], inp["B"], inp["s"], amax_x=amax_x, qw=qw)
    oracle.linear_bwd(dY, X, Wr, U, V, inp["A"], inp["B"], inp["s"], f["P"], amax_dy=amax_dy, qw=qw)


def oracle_workload(workload, inputs=None):
    """[(shape, inputs, prep)] of the linears one oracle step covers: the
    four linear types of a DiT block (every block has the same shapes and
    work) or the attention projection.  `inputs`: the already drawn
    make_inputs dicts, one per linear type (else drawn here)."""
    import ft_synth
    shapes = stack_shapes() if workload == "dit8" else [ft_synth.ATTN]
    seeds = [SEED + j for j in range(len(shapes))] if workload == "dit8" else [1]
    out = []
    for i, (sh, sd) in enumerate(zip(shapes, seeds)):
        inp = inputs[i] if inputs is not None else ft_synth.make_inputs(sh, seed=sd)
        out.append((sh, inp, oracle_prep(sh, inp)))
    return out


def oracle_steps(items, rows_per_linear, n, rng, seconds=None):
    """Runs oracle steps (each linear on its own random row sample); returns
    per-step (seconds, FP4 GEMM FLOP the sample stands for)."""
    res = []
    t_total = 0.0
    for _ in range(n):
        t0 = time.perf_counter()
        flops = 0.0
        for sh, inp, prep in items:
            rows = np.sort(rng.choice(sh.M, rows_per_linear, replace=False))
            oracle_sample_step(inp, prep, rows)
            flops += gemm_flops(sh, rows_per_linear)
        dt = time.perf_counter() - t0
        res.append((dt, flops))
        t_total += dt
        if seconds is not None and t_total >= seconds:
            break
    return res


def cpu_baseline(workload, items, rows_per_linear, seconds=15.0):
    """Times the oracle as it stands on the host cores over a bounded sample."""
    res = oracle_steps(items, rows_per_linear, 64, np.random.default_rng(123), seconds=seconds)
    t = sum(r[0] for r in res)
    fl = sum(r[1] for r in res)
    what = "the four linears of one DiT block" if workload == "dit8" else "the attention projection"
    return {
        "value": fl / t / 1e12,
        "unit": UNIT,
        "cores": blas_threads(),
        "kind": "oracle",
        "sample": f"{len(res)} oracle steps, each the fwd+bwd of {what} on {rows_per_linear} random token "
                  f"rows per linear (tensor scales from the full tensors; every block of the stack has "
                  f"the same shapes), {t:.1f} s of host time; FLOP/s of the sample",
    }


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    items = oracle_workload(args.workload)
    rng = np.random.default_rng(7)
    R = args.sample_rows
    oracle_steps(items, R, args.warmup, rng)
    res = oracle_steps(items, R, args.steps, rng)
    t_step = sum(r[0] for r in res) / len(res)
    value = sum(r[1] for r in res) / sum(r[0] for r in res) / 1e12
    what = "the four linears of one DiT block" if args.workload == "dit8" else "the attention projection"
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
        "config": {"workload": workload_name(args.workload) + f"; oracle step = fwd+bwd of {what} on "
                                                              f"{R} random token rows per linear",
                   "global_batch": R, "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: fwd+bwd of {what} on {R} random token rows per linear"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


def workload_name(workload):
    if workload == "dit8":
        return ("dit8: 8-block DiT linear stack (hidden 3072, MLP 12288), per block QKV [9216,3072], "
                "out [3072,3072], up [12288,3072], down [3072,12288]; M=4608 tokens; stabilizer rank 32, "
                "LoRA rank 32; fwd of all 32 linears then bwd (dgrad + LoRA grads) in reverse")
    return ("attn_proj: X [4608,3072] bf16 (1% outlier channels x30), W [3072,3072], stabilizer rank 32, "
            "LoRA rank 16; fwd + dgrad + LoRA grads")


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


def ncu_traffic(kernel: str, source: str, key: str | None = None):
    """DRAM bytes per launch from the committed ncu summary, when it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[key or kernel]
        if e.get("source_sha") == kernel_source_sha(source):
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def quant_bytes(M, C, r):
    """Algorithmic bytes of one fused quantize + down-projection of T [M, C]:
    read T and the [C, r] factors, write codes (0.5 B), scales (1/16 B) and
    P [M, r] bf16."""
    return M * C * (2 + 0.5 + 1 / 16) + C * r * 2 + M * r * 2


def lora_grad_bytes(M, N, K, r):
    """Algorithmic bytes of the adapter gradients: read dY [M, N] and X
    [M, K] (bf16) and the saved P, Pg [M, r] bf16 (the outputs are small)."""
    return M * (N + K) * 2 + 2 * M * r * 2


def call_work(L, M, direction, kernel):
    """Algorithmic work of one launch of `kernel` inside one call: FLOP for
    the GEMM, bytes for the bandwidth-bound kernels."""
    r = L.r_s + L.r_l
    C = L.K if direction == "fwd" else L.N
    if kernel == "k_gemm_fp4":
        return 2.0 * M * L.N * L.K
    if kernel in ("k_qres", "k_qdown"):
        return quant_bytes(M, C, r)
    if kernel == "k_amax_bf16":
        return M * C * 2.0
    if kernel == "k_lora_grad":
        return lora_grad_bytes(M, L.N, L.K, r)
    return None


class Flush:
    """L2 flush between steps: write a buffer larger than the 126 MB L2, then
    read another one, so each step starts with a cold L2 that holds neither
    the step's data nor dirty lines awaiting write-back."""

    def __init__(self, torch, dev):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def keep_host_ahead(torch, ms=3):
    """A short device-side sleep so the whole step is enqueued before the GPU
    reaches it: the step's events then time device work only."""
    torch.cuda._sleep(int(ms * 1_000_000))


def timed_steps(torch, step, steps, warmup, flush, dist, sleep_ms=3):
    """W warm-up steps, then K steps each bracketed by CUDA events on the
    current stream (the L2 flush and the device sleep outside the events);
    returns (per-step ms, wall seconds, clock record)."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()).start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    evs = []
    for _ in range(steps):
        flush()
        keep_host_ahead(torch, sleep_ms)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    wall = time.perf_counter() - t0
    clocks = sampler.stop()
    return [a.elapsed_time(b) for a, b in evs], wall, clocks


def kernel_pass(torch, ft, calls, steps, flush):
    """The same calls again with every library launch bracketed by CUDA
    events on its stream; `calls` is [(key, fn)] of one step.  Returns
    {(key, kernel): [ms, launches]} summed over the steps and the launches
    per step."""
    acc = {}
    ft.timing.reset()
    ft.timing.enable(True)
    prev = {k: (0.0, 0) for k in KERNELS}
    total = 0
    for _ in range(steps):
        flush()
        keep_host_ahead(torch)
        for key, fn in calls:
            fn()
            for k in KERNELS:
                ms, n = ft.timing.read(k)
                dms, dn = ms - prev[k][0], n - prev[k][1]
                prev[k] = (ms, n)
                if dn:
                    a = acc.setdefault((key, k), [0.0, 0])
                    a[0] += dms
                    a[1] += dn
                    total += dn
    torch.cuda.synchronize()
    ft.timing.enable(False)
    return acc, total // steps


def summarize_kernels(acc, layer_of, M):
    """Per kernel: launches, ms, and the achieved rate over the step's
    launches (algorithmic work / event time)."""
    out = {}
    for (key, k), (ms, n) in acc.items():
        L, direction = layer_of[key]
        w = call_work(L, M, direction, k)
        e = out.setdefault(k, {"ms": 0.0, "launches": 0, "work": 0.0, "by_call": {}})
        e["ms"] += ms
        e["launches"] += n
        if w is not None:
            e["work"] += w * n
        e["by_call"][key] = {"us_per_launch": ms / n * 1e3, "launches": n,
                             "work_per_launch": w}
    for k, e in out.items():
        e["rate"] = e["work"] / (e["ms"] * 1e-3) if e["work"] else None
    return out


def clone_layer(ft, L):
    """A copy of a prepared layer in its own device memory (the blocks of the
    stack hold their own weights)."""
    import dataclasses

    def c(t):
        return None if t is None else t.clone()

    def cf(f):
        return ft.FP4(c(f.codes), c(f.scales), c(f.tscale), f.rows, f.cols, f.blk)

    w_k = cf(L.w_k)
    w_n = ft.FP4(c(L.w_n.codes), w_k.scales, w_k.tscale, L.w_n.rows, L.w_n.cols, L.w_n.blk)
    return dataclasses.replace(L, w_k=w_k, w_n=w_n, U=c(L.U), V=c(L.V), A=c(L.A), B=c(L.B),
                               op_k=c(L.op_k), op_n=c(L.op_n))


def bench_quantizers(torch, ft, dev, hbm_gbs, flush, reps=10):
    """The standalone quantize kernels (the GB/s-against-HBM half of the
    metric): per case
    the algorithmic bytes of one call, its time (CUDA events around the call,
    L2 flushed before each) and the fraction of the HBM peak.  'supplied'
    runs take the tensor amax from the caller (single pass); 'computed' runs
    find it themselves (the two-pass streaming path re-reads the input: its
    two_pass_bytes count that read)."""
    import ft_synth

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(dev).view(torch.bfloat16)

    a = ft_synth.make_inputs(ft_synth.ATTN, seed=1, M=4608)
    X_attn = to_dev(a["X"])
    d = ft_synth.make_inputs(ft_synth.MLP_UP, seed=2)
    dY_up = to_dev(d["dY"])
    X_dn = to_dev(ft_synth.make_inputs(ft_synth.MLP_DOWN, seed=3)["X"])
    W_up = to_dev(d["W"])
    amax = {id(t): t.abs().max().float().reshape(1) for t in (X_attn, dY_up, X_dn, W_up)}
    ws = ft.Workspace()
    cases = []
    # (name, tensor, fn(amax or None), bytes per element of the single-pass
    # definition); outputs allocated once, outside the timed calls
    for t, nm in ((X_attn, "X [4608,3072]"), (X_dn, "X [4608,12288]")):
        o = ft.FP4.empty(t.shape[0], t.shape[1], ft.BLK_1x16, dev)
        cases.append((f"ft_quantize 1x16 {nm}", t,
                      lambda am, t=t, o=o: ft.ft_quantize(t, ft.BLK_1x16, amax=am, out=o, ws=ws), 2.5625))
    for t, nm in ((X_attn, "X [4608,3072]"), (dY_up, "dY [4608,12288]")):
        o_r = ft.FP4.empty(t.shape[0], t.shape[1], ft.BLK_1x16, dev)
        o_c = ft.FP4.empty(t.shape[1], t.shape[0], ft.BLK_1x16, dev)
        cases.append((f"ft_quantize_transpose 1x16 {nm}", t,
                      lambda am, t=t, o_r=o_r, o_c=o_c: ft.ft_quantize_transpose(
                          t, ft.BLK_1x16, amax=am, out_row=o_r, out_col=o_c, ws=ws), 3.125))
    w_r = ft.FP4.empty(W_up.shape[0], W_up.shape[1], ft.BLK_16x16, dev)
    w_c = ft.FP4.empty(W_up.shape[1], W_up.shape[0], ft.BLK_16x16, dev, scales=w_r.scales, tscale=w_r.tscale)
    cases.append(("ft_quantize_transpose 16x16 W [12288,3072]", W_up,
                  lambda am: ft.ft_quantize_transpose(W_up, ft.BLK_16x16, amax=am, out_row=w_r, out_col=w_c,
                                                      ws=ws), 3.0 + 1 / 256))
    stream = torch.cuda.current_stream()
    out = {}
    for name, t, fn, bpe in cases:
        for mode in ("supplied", "computed"):
            am = amax[id(t)] if mode == "supplied" else None
            fn(am)
            torch.cuda.synchronize()
            ms = []
            ft.timing.reset()
            ft.timing.enable(True)
            for _ in range(reps):
                flush()
                keep_host_ahead(torch, 0.5)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn(am)
                e1.record(stream)
                e1.synchronize()
                ms.append(e0.elapsed_time(e1))
            ft.timing.enable(False)
            kern = {k: ft.timing.read(k) for k in KERNELS}
            used = {k: round(v[0] / v[1] * 1e3, 2) for k, v in kern.items() if v[1]}
            t_ms = statistics.median(ms)
            nbytes = t.numel() * bpe
            two_pass = mode == "computed" and "k_amax_bf16" in used
            e = {"bytes": nbytes, "us": t_ms * 1e3, "gbs": nbytes / (t_ms * 1e-3) / 1e9,
                 "frac": nbytes / (t_ms * 1e-3) / 1e9 / hbm_gbs, "kernels_us": used}
            if two_pass:
                tb = nbytes + t.numel() * 2
                e["two_pass_bytes"] = tb
                e["two_pass_frac"] = tb / (t_ms * 1e-3) / 1e9 / hbm_gbs
            out[f"{name} ({mode} amax)"] = e
    assert ft.ft_device_error() == 0, "device error in the quantizer section"
    return out


def run_attn_secondary(torch, ft, dev, flush, steps, warmup, fp4_peak, hbm_gbs):
    """The attention projection alone (one linear, fwd + bwd): step rate, the
    GEMM's and the quantizer's fractions."""
    import ft_synth
    shape = ft_synth.ATTN

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(dev).view(torch.bfloat16)

    inp = ft_synth.make_inputs(shape, seed=1)
    X, dY = to_dev(inp["X"]), to_dev(inp["dY"])
    layer = ft.prepare_layer(to_dev(inp["W"]), shape.r_s, A=to_dev(inp["A"]), B=to_dev(inp["B"]), s=inp["s"])
    from bit_quantized_lora_b200.stack import LinearStack
    st = LinearStack([layer], shape.M, dev)
    ms, _, _ = timed_steps(torch, lambda: st.step([X], [dY]), steps, warmup, flush, None, sleep_ms=2)
    calls = [("attn.fwd", lambda: st.forward_layer(0, X)), ("attn.bwd", lambda: st.backward_layer(0, dY, X))]
    acc, _ = kernel_pass(torch, ft, calls, steps, flush)
    ks = summarize_kernels(acc, {"attn.fwd": (layer, "fwd"), "attn.bwd": (layer, "bwd")}, shape.M)
    step_ms = sum(ms) / len(ms)
    res = {"workload": workload_name("attn_proj"), "ms_per_step": step_ms,
           "value": gemm_flops(shape) / (step_ms * 1e-3) / 1e12, "unit": UNIT}
    if "k_gemm_fp4" in ks:
        g = ks["k_gemm_fp4"]["rate"] / 1e12
        res["gemm"] = {"achieved": g, "frac": g / fp4_peak, "unit": "TFLOP/s",
                       "launch_us": ks["k_gemm_fp4"]["ms"] / ks["k_gemm_fp4"]["launches"] * 1e3}
    if "k_qres" in ks:
        q = ks["k_qres"]["rate"] / 1e9
        res["k_qres"] = {"achieved": q, "frac": q / hbm_gbs, "unit": "GB/s",
                         "launch_us": ks["k_qres"]["ms"] / ks["k_qres"]["launches"] * 1e3}
    if "k_lora_grad" in ks:
        q = ks["k_lora_grad"]["rate"] / 1e9
        res["k_lora_grad"] = {"achieved": q, "frac": q / hbm_gbs, "unit": "GB/s"}
    return res


def bench_mlp(torch, ft, dev, flush, reps=10):
    """MLP fusion (the FourTune page's section 3.3; its Fig. 9 credits it
    with a further 1.10x): one DiT block's MLP forward, X [4608, 3072] ->
    up [12288, 3072] -> GELU -> down [3072, 12288], fused (FC1's GEMM
    epilogue applies GELU and quantizes H for FC2 with a supplied tensor
    amax) against the same calls unfused (FC1, the GELU kernel, FC2 with its
    own quantizer, with the amax supplied or computed).  CUDA events around
    each forward, L2 flushed before each."""
    import ft_synth
    sh_up, sh_dn = stack_shapes()[2], stack_shapes()[3]

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(dev).view(torch.bfloat16)

    iu = ft_synth.make_inputs(sh_up, seed=SEED + 2)
    wd = ft_synth.make_inputs(dataclasses_replace(sh_dn, M=16), seed=SEED + 3)
    up = ft.prepare_layer(to_dev(iu["W"]), sh_up.r_s, A=to_dev(iu["A"]), B=to_dev(iu["B"]), s=iu["s"])
    dn = ft.prepare_layer(to_dev(wd["W"]), sh_dn.r_s, A=to_dev(wd["A"]), B=to_dev(wd["B"]), s=wd["s"])
    X = to_dev(iu["X"])
    M = sh_up.M
    Y_up, _ = ft.ft_linear_fwd(up, X)
    H = ft.ft_gelu_bf16(Y_up)
    amax_h = H.abs().max().float().reshape(1)
    ws_f, ws_u = ft.Workspace(), ft.Workspace()
    Yd = torch.empty(M, sh_dn.N, dtype=torch.bfloat16, device=dev)
    Pu = torch.empty(M, sh_up.r_s + sh_up.r_l, dtype=torch.bfloat16, device=dev)
    Pd = torch.empty(M, sh_dn.r_s + sh_dn.r_l, dtype=torch.bfloat16, device=dev)
    Hf = torch.empty_like(H)

    def fused():
        ft.ft_mlp_fwd(up, dn, X, amax_h, H=Hf, Y=Yd, P_up=Pu, P_down=Pd, ws=ws_f)

    def unfused(amax):
        ft.ft_linear_fwd(up, X, Y=Y_up, P=Pu, ws=ws_u)
        ft.ft_gelu_bf16(Y_up, out=H)
        ft.ft_linear_fwd(dn, H, amax_x=amax, Y=Yd, P=Pd, ws=ws_u)

    stream = torch.cuda.current_stream()
    out = {}
    for name, fn in (("fused", fused), ("unfused_supplied_amax", lambda: unfused(amax_h)),
                     ("unfused_computed_amax", lambda: unfused(None))):
        fn()
        torch.cuda.synchronize()
        ms = []
        ft.timing.reset()
        ft.timing.enable(True)
        for _ in range(reps):
            flush()
            keep_host_ahead(torch, 1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        ft.timing.enable(False)
        out[name + "_ms"] = statistics.median(ms)
        kern = {k: ft.timing.read(k) for k in KERNELS}
        # per forward: the summed time of each kernel's launches in it
        out[name + "_kernels_us"] = {k: round(v[0] / reps * 1e3, 2) for k, v in kern.items() if v[1]}
    assert ft.ft_device_error() == 0, "device error in the MLP section"
    out["speedup_vs_unfused_supplied"] = out["unfused_supplied_amax_ms"] / out["fused_ms"]
    out["speedup_vs_unfused_computed"] = out["unfused_computed_amax_ms"] / out["fused_ms"]
    out["workload"] = "X [4608,3072] -> up [12288,3072] -> GELU -> down [3072,12288], r_s = r_l = 32, bf16 outputs"
    return out


def bench_lora_fusion(torch, ft, dev, flush, reps=10):
    """LoRA fusion (the FourTune page's section 3.3; its Fig. 9 credits it
    with 1.82x): one forward of the DiT MLP-up linear (X [4608, 3072],
    W [12288, 3072], r_s = r_l = 32, bf16 Y) as the library runs it -- P =
    [X U | s X A] made by the quantizer's pass over X, P [V | B]^T added in
    the GEMM's epilogue, Y written once -- against the same layer unfused:
    the 4-bit GEMM alone (rank 0, FP32 Y), then the low-rank branch as
    separate bf16 matmuls (torch), the add and the cast to bf16.  CUDA events
    around each forward, L2 flushed before each."""
    import ft_synth
    sh = stack_shapes()[2]

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(dev).view(torch.bfloat16)

    inp = ft_synth.make_inputs(sh, seed=SEED + 2)
    U, V, Wr = ft.svd_split(to_dev(inp["W"]), sh.r_s)
    A, B, s = to_dev(inp["A"]), to_dev(inp["B"]), float(inp["s"])
    fused = ft.prepare_layer(W_res=Wr, U=U, V=V, A=A, B=B, s=s)
    bare = ft.prepare_layer(W_res=Wr)
    X = to_dev(inp["X"])
    M, N = X.shape[0], Wr.shape[0]
    r = U.shape[1] + A.shape[1]
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    P = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    Y32 = torch.empty(M, N, dtype=torch.float32, device=dev)
    UA = torch.cat([U, A * s], dim=1).contiguous()   # [K, r], s folded into A
    LR = torch.cat([V, B], dim=1).contiguous()       # [N, r]
    ws_f, ws_b = ft.Workspace(), ft.Workspace()

    def run_fused():
        ft.ft_linear_fwd(fused, X, Y=Y, P=P, ws=ws_f)

    def run_unfused():
        ft.ft_linear_fwd(bare, X, out_dtype=ft.F32, Y=Y32, ws=ws_b)
        Pu = X @ UA
        Y32.add_(Pu @ LR.T)
        Y.copy_(Y32)

    stream = torch.cuda.current_stream()
    out = {}
    for name, fn in (("fused", run_fused), ("unfused", run_unfused)):
        fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(reps):
            flush()
            keep_host_ahead(torch, 1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        out[name + "_ms"] = statistics.median(ms)
    assert ft.ft_device_error() == 0, "device error in the LoRA-fusion section"
    out["speedup"] = out["unfused_ms"] / out["fused_ms"]
    out["workload"] = ("X [4608,3072], W [12288,3072], r_s = r_l = 32, bf16 Y; unfused = rank-0 4-bit GEMM (FP32 Y) "
                       "+ torch bf16 matmuls X [U | sA], P [V | B]^T + add + cast")
    return out


def dataclasses_replace(obj, **kw):
    import dataclasses
    return dataclasses.replace(obj, **kw)


def run_ours(args):
    import torch

    import ft_synth
    import bit_quantized_lora_b200 as ft
    from bit_quantized_lora_b200 import dp
    from bit_quantized_lora_b200.stack import LinearStack

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    group = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    hbm_gbs, bf16_tflops, bf16_sustained, peak_src = measured_peaks()

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(dev).view(torch.bfloat16)

    # ---------------- synthetic inputs (weak scaling): the weights are
    # replicas (one seed per linear type for every rank); every rank owns its
    # own batch of tokens
    if args.workload == "dit8":
        shapes = stack_shapes()
        seeds = [SEED + j for j in range(len(shapes))]
        n_blocks = N_BLOCKS
    else:
        shapes = [ft_synth.ATTN]
        seeds = [1]
        n_blocks = 1
    M = shapes[0].M
    base_layers, host_tok, drawn = [], [], []
    for sh, sd in zip(shapes, seeds):
        wts = ft_synth.make_inputs(sh, seed=sd)
        tok = wts if dp.rank_seed(sd, rank) == sd else ft_synth.make_inputs(sh, seed=dp.rank_seed(sd, rank))
        # untimed preparation: SVD split, 16x16 quantization, operand images
        base_layers.append(ft.prepare_layer(to_dev(wts["W"]), sh.r_s, A=to_dev(wts["A"]), B=to_dev(wts["B"]),
                                            s=wts["s"]))
        host_tok.append((tok["X"], tok["dY"]))
        drawn.append(wts if tok is wts else None)
    layers, Xs, dYs, layer_of, keys = [], [], [], {}, []
    for b in range(n_blocks):
        for j, sh in enumerate(shapes):
            L = base_layers[j] if b == 0 else clone_layer(ft, base_layers[j])
            layers.append(L)
            # each block's linear has its own input buffers (the same seeded draws)
            Xs.append(to_dev(host_tok[j][0]))
            dYs.append(to_dev(host_tok[j][1]))
            key = sh.name.split(".", 1)[-1] if n_blocks > 1 else sh.name
            keys.append(key)
            layer_of[key + ".fwd"] = (L, "fwd")
            layer_of[key + ".bwd"] = (L, "bwd")
    stack = LinearStack(layers, M, dev)
    flush = Flush(torch, dev)

    def step():
        stack.step(Xs, dYs, group)

    step()
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0, "device error in the first step"

    # ---------------- timed region (kernel inputs resident in HBM); the
    # library's per-kernel events stay off here and are taken in a separate
    # pass below, so they add nothing between the step's launches
    step_ms, t_wall, clocks = timed_steps(torch, step, args.steps, args.warmup, flush, dist)
    assert ft.ft_device_error() == 0, "device error during the timed region"
    ms_step = dp.max_over_ranks(sum(step_ms) / len(step_ms), dev)

    # ---------------- per-kernel durations: the same calls (without the
    # exchange), each library launch bracketed by CUDA events on its stream
    calls = [(keys[j] + ".fwd", lambda j=j: stack.forward_layer(j, Xs[j])) for j in range(len(layers))]
    calls += [(keys[j] + ".bwd", lambda j=j: stack.backward_layer(j, dYs[j], Xs[j]))
              for j in reversed(range(len(layers)))]
    kpass_steps = max(2, min(args.steps, 5))
    acc, launches_per_step = kernel_pass(torch, ft, calls, kpass_steps, flush)
    assert ft.ft_device_error() == 0, "device error during the per-kernel pass"
    ks = summarize_kernels(acc, layer_of, M)

    flops = sum(gemm_flops(sh) for sh in shapes) * n_blocks
    value = dp.job_rate(flops, world, ms_step) / 1e12
    # the burst peak unless the clocks show the power cap engaged during the
    # timed region (then the sustained figure, measured under that cap)
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    bf16_peak = bf16_sustained if (capped and bf16_sustained) else bf16_tflops
    fp4_peak = bf16_peak * FP4_OVER_BF16

    g = ks["k_gemm_fp4"]
    gemm_achieved = g["rate"] / 1e12
    per_kernel = {}
    for k, e in ks.items():
        ent = {"launches_per_step": e["launches"] / kpass_steps, "ms_per_step": e["ms"] / kpass_steps}
        if e["rate"] is not None:
            if k == "k_gemm_fp4":
                ent.update({"achieved": e["rate"] / 1e12, "unit": "TFLOP/s", "frac": e["rate"] / 1e12 / fp4_peak})
            else:
                ent.update({"achieved": e["rate"] / 1e9, "unit": "GB/s", "frac": e["rate"] / 1e9 / hbm_gbs})
        ent["us_per_launch_by_call"] = {c: round(v["us_per_launch"], 2) for c, v in e["by_call"].items()}
        per_kernel[k] = ent

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
        "data": "synthetic (seeded; FLUX-like DiT shapes, random-init weights; every block holds its own copy "
                "of the same seeded draws)",
        "config": {
            "workload": workload_name(args.workload),
            "global_batch": M * world,
            "seq_len": M,
            "parallelism": f"dp{world}" if world > 1 else "single",
            "gemm_tiling": "CTA pairs, 256 x 256 tiles" if args.gemm_mode == "pairs" else "one CTA per 128 x 256 tile",
            "l2": "inputs larger than L2 (the step touches several GB) and flushed between steps "
                  "(256 MB write then 256 MB read, outside the step events)",
        },
        "roofline": {
            "kernel": "k_gemm_fp4",
            "bound": "tensor",
            "achieved": gemm_achieved,
            "peak": fp4_peak,
            "unit": "TFLOP/s",
            "frac": gemm_achieved / fp4_peak,
            "traffic": ncu_traffic("k_gemm_fp4", "k_gemm_fp4.cuh", "k_gemm_fp4@dit8"),
            "peak_source": f"{peak_src} bf16 {'sustained' if bf16_peak != bf16_tflops else 'burst'} "
                           f"{bf16_peak} TFLOP/s x {FP4_OVER_BF16} (nominal NVFP4/bf16)",
            "flop_per_step": g["work"] / kpass_steps,
            "launches_per_step": g["launches"] / kpass_steps,
            "note": "achieved = the step's GEMM FLOP / the summed CUDA-event time of its GEMM launches",
        },
        "kernels": per_kernel,
        "gpu_launches": launches_per_step * args.steps,
        "wall_s_timed_region": t_wall,
        "clocks": clocks,
    }
    if dist is None and not args.skip_extras:
        out["attn_proj"] = run_attn_secondary(torch, ft, dev, flush, args.steps, args.warmup, fp4_peak, hbm_gbs)
        out["quantize"] = bench_quantizers(torch, ft, dev, hbm_gbs, flush)
        out["mlp_fusion"] = bench_mlp(torch, ft, dev, flush)
        out["lora_fusion"] = bench_lora_fusion(torch, ft, dev, flush)

    # ---------------- end to end through the API with host buffers: every
    # linear's X and dY copied in from pinned host memory, the step, and the
    # step's result -- the adapter gradients of every layer, what a training
    # step hands to the optimizer -- read back.  Y and dX stay on the device:
    # in a training step the neighbouring layers consume them there.  The
    # copies run on their own stream in the order the step consumes them
    # (the X of each layer, then the dY of each layer from the last), and
    # each layer waits only for its own inputs, as an input pipeline would
    # overlap them; all of them lie inside the timed region.
    if not args.skip_extras:
        pinned = [(torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory(),
                   torch.from_numpy(np.ascontiguousarray(d).view(np.int16)).view(torch.bfloat16).pin_memory())
                  for x, d in host_tok]
        gh = torch.empty(stack.grads.numel(), dtype=torch.float32).pin_memory()
        stream = torch.cuda.current_stream()
        copy_stream = torch.cuda.Stream(device=dev)
        xev = [torch.cuda.Event() for _ in layers]
        dyev = [torch.cuda.Event() for _ in layers]
        e2e_ms = []
        if dist is not None:
            dist.barrier()
        nsh = len(shapes)
        for i in range(args.warmup + args.steps):
            flush()
            keep_host_ahead(torch)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            copy_stream.wait_event(e0)
            with torch.cuda.stream(copy_stream):
                for j in range(len(layers)):
                    Xs[j].copy_(pinned[j % nsh][0], non_blocking=True)
                    xev[j].record(copy_stream)
                for j in reversed(range(len(layers))):
                    dYs[j].copy_(pinned[j % nsh][1], non_blocking=True)
                    dyev[j].record(copy_stream)
            stack.step(Xs, dYs, group, x_ready=xev, dy_ready=dyev)
            gh.copy_(stack.grads, non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            if i >= args.warmup:
                e2e_ms.append(e0.elapsed_time(e1))
        ms_e2e = dp.max_over_ranks(sum(e2e_ms) / len(e2e_ms), dev)
        out["e2e"] = {
            "value": dp.job_rate(flops, world, ms_e2e) / 1e12,
            "unit": UNIT,
            "h2d_bytes_per_step": sum(x.numel() * 2 + d.numel() * 2 for x, d in zip(Xs, dYs)),
            "d2h_bytes_per_step": stack.grads.numel() * 4,
            "ms_per_step": ms_e2e,
        }
    assert ft.ft_device_error() == 0, "device error after the end-to-end leg"
    if world == 1 and rank == 0 and not args.skip_cpu_baseline:
        reuse = drawn if all(d is not None for d in drawn) else None
        out["cpu_baseline"] = cpu_baseline(args.workload, oracle_workload(args.workload, reuse), args.sample_rows)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


def run_single(args):
    """One linear of the DiT stack, forward then backward, --steps times: a
    short, fixed launch sequence for ncu captures (per step: the input's
    quantizer -- k_qres, or k_amax_bf16 + k_qdown --, the forward GEMM, the
    output gradient's quantizer, the dgrad GEMM, k_lora_grad).  With
    "mlp": one DiT block's fused MLP forward per step (k_qres of X, FC1's
    GEMM with the GELU + Q(H) epilogue, k_qdown's P-only pass over H, FC2's
    GEMM)."""
    import torch

    import ft_synth
    import bit_quantized_lora_b200 as ft
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.single == "mlp":
        return run_single_mlp(args, torch, ft, dev)
    j = ["qkv", "out", "up", "down"].index(args.single)
    sh = stack_shapes()[j]
    inp = ft_synth.make_inputs(sh, seed=SEED + j)

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(dev).view(torch.bfloat16)

    layer = ft.prepare_layer(to_dev(inp["W"]), sh.r_s, A=to_dev(inp["A"]), B=to_dev(inp["B"]), s=inp["s"])
    from bit_quantized_lora_b200.stack import LinearStack
    st = LinearStack([layer], sh.M, dev)
    X, dY = to_dev(inp["X"]), to_dev(inp["dY"])
    for _ in range(args.steps):
        st.step([X], [dY])
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0, "device error"
    print("ok", flush=True)
    return 0


def run_single_mlp(args, torch, ft, dev):
    import ft_synth
    sh_up, sh_dn = stack_shapes()[2], stack_shapes()[3]

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(dev).view(torch.bfloat16)

    iu = ft_synth.make_inputs(sh_up, seed=SEED + 2)
    wd = ft_synth.make_inputs(dataclasses_replace(sh_dn, M=16), seed=SEED + 3)
    up = ft.prepare_layer(to_dev(iu["W"]), sh_up.r_s, A=to_dev(iu["A"]), B=to_dev(iu["B"]), s=iu["s"])
    dn = ft.prepare_layer(to_dev(wd["W"]), sh_dn.r_s, A=to_dev(wd["A"]), B=to_dev(wd["B"]), s=wd["s"])
    X = to_dev(iu["X"])
    # H's tensor amax from one unfused FC1 + GELU (one k_gemm_fp4 launch
    # before the loop's)
    Y_up, _ = ft.ft_linear_fwd(up, X)
    amax_h = ft.ft_gelu_bf16(Y_up).abs().max().float().reshape(1)
    del Y_up
    ws = ft.Workspace()
    for _ in range(args.steps):
        ft.ft_mlp_fwd(up, dn, X, amax_h, ws=ws)
    torch.cuda.synchronize()
    assert ft.ft_device_error() == 0, "device error"
    print("ok", flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.gemm_mode == "single":
        import bit_quantized_lora_b200 as ft
        ft.ft_set_gemm_mode(ft.GEMM_SINGLE)
    if args.single:
        return run_single(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
