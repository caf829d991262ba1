#!/usr/bin/env python3
"""Benchmark of the W8A8 int8-dynamic linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qkv|ffn_up|ffn_down|adaln_m1|adaln_m2|adaln_m16]
                    [--no-extras] [--no-sweep] [--no-e2e] [--no-cpu-baseline]
                    [--cpu-budget S]

A step is one whole layer call on one batch: per-token quantization of the
bf16 activations, the int8 tensor-core GEMM and the fused dequantization
epilogue (w8a8_linear_fused).  The headline workload is the DiT fused-QKV
projection, x [4352, 3072] (4096 image + 256 text tokens) against W [9216, 3072].
Weights are quantized once before timing (load time).  The metric is int8
TOPS = 2*M*N*K / time of the whole layer (quantization included).

Timing: W warm-up steps, then K steps bracketed by a barrier and a device
synchronize on both sides, timed with CUDA events on the launching stream;
the reported time is the max over ranks.  Between steps the inputs rotate
over several independent buffer sets whose combined size exceeds twice the
126 MB L2, so no step reads data a previous step left in L2.

Beside the headline line's own figures (roofline of the dominant kernel,
end-to-end time from pinned host buffers, CPU oracle baseline, clocks sampled
during the timed region), `components` reports the other workloads: the
AdaLN GEMV at M = 1 and 2, the FFN layers alone and back to back, one DiT
block's linears at CFG batch 2, the small-M regime, the M sweep over the
block's four linear shapes (32 points), packed-weight loading and the W8A16
variant.  The roofline's denominator is measured in the same run: the
tcgen05 kind::i8 instruction issued back to back on every CTA pair with no
memory traffic; torch._int_mm at 8192^3 is reported beside it as the
library's rate.

Multi-GPU: the layer shards into independent problems, so N ranks run N
replicas with no collective on the data path (weak scaling); `value` is the
sum over ranks.  One rank per GPU: `--gpus N` started without a launcher
re-executes itself under torchrun with N ranks; under torchrun it reads
RANK / LOCAL_RANK / WORLD_SIZE.  At N > 1 the extra components are skipped.

--impl reference times the CPU oracle (plain C, OpenMP) on rank 0 on a
bounded row sample of the same workload; the other ranks exit without work.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
NOMINAL_INT8_TOPS = 4500.0           # dense int8, B200 datasheet
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
WORKLOADS = {"qkv": synth.QKV, "ffn_up": synth.FFN_UP, "ffn_down": synth.FFN_DOWN,
             "adaln_m1": synth.ADALN_M1, "adaln_m2": synth.ADALN_M2,
             "adaln_m16": synth.ADALN_M16}


# ----------------------------------------------------------------------------- utils

def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def bf16_dev(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def n_sets(bytes_per_set: int) -> int:
    """Buffer sets to rotate so the other sets total more than 2x L2."""
    return max(3, math.ceil(2 * L2_BYTES / max(bytes_per_set, 1)) + 1)


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.ok = False
        self.samples, self.reasons = [], 0
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that, do not guess
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            # the launching thread holds the GIL most of the time: hand it
            # over more often so the sampler runs at its period
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(2e-4)
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            sys.setswitchinterval(self._switch)

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def profile_traffic(kernel_tag: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel, or
    None when the summary is absent or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    try:
        text = open(path).read()
    except OSError:
        return None, None
    m = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{16,64})", text)
    if not m:
        return None, None
    if h and h.group(1) != kernel_source_hash(kernel_tag)[: len(h.group(1))]:
        return None, "stale"
    return float(m.group(1)), "ncu"


# The device source files each profiled kernel is built from.
KERNEL_SOURCES = {
    "gemm_i8_tcgen05": ("w8a8_gemm.cuh", "w8a8_ptx.cuh", "w8a8_quant.cuh"),
    "gemv_i8": ("w8a8_gemv.cuh", "w8a8_prefetch.cuh", "w8a8_ptx.cuh", "w8a8_quant.cuh"),
    "gemm_i8_swapab": ("w8a8_swapab.cuh", "w8a8_gemm.cuh", "w8a8_ptx.cuh"),
    "quant_rows": ("w8a8_quant.cuh", "w8a8_ptx.cuh"),
}


def kernel_source_hash(kernel_tag: str = "") -> str:
    """sha256 of the device sources of the kernel a profile tag names (all of
    them for an unknown tag)."""
    d = os.path.join(ROOT, "w8a8_int8_dynamic_token_b200", "csrc")
    names = next((v for k, v in KERNEL_SOURCES.items() if kernel_tag.startswith(k)), None)
    if names is None:
        names = [n for n in os.listdir(d) if n.endswith((".cu", ".cuh"))]
    hs = hashlib.sha256()
    for name in sorted(names):
        with open(os.path.join(d, name), "rb") as f:
            hs.update(f.read())
    return hs.hexdigest()


# ----------------------------------------------------------------------------- our arm

class Layer:
    """One workload's device buffers, rotated over several independent sets."""

    def __init__(self, case: synth.LayerCase, device, with_ws=True, x_bits=None, weights=None):
        """weights: (Wq, s_w) already quantized on the device, to share one
        weight between several layers of the same (K, N); x_bits: the host
        activations when the caller has generated them already."""
        import w8a8_int8_dynamic_token_b200 as w8a8
        self.w8a8 = w8a8
        self.case = case
        M, K, N = case.M, case.K, case.N
        x_bits = case.x() if x_bits is None else x_bits
        b_bits = case.b()
        x0 = bf16_dev(x_bits, device)
        if weights is None:
            W = bf16_dev(case.w(), device)
            Wq, s_w = w8a8.quantize_weights(W)      # load-time weight quantization
            del W
        else:
            Wq, s_w = weights
        b0 = bf16_dev(b_bits, device) if b_bits is not None else None
        self.ws_bytes = w8a8.workspace_size(M, N, K) if with_ws else 0
        per_set = 2 * M * K + N * K + 6 * N + 2 * M * N + self.ws_bytes
        self.sets = []
        for _ in range(n_sets(per_set)):
            self.sets.append({
                "x": x0.clone(), "Wq": Wq.clone(), "s_w": s_w.clone(),
                "b": b0.clone() if b0 is not None else None,
                "y": torch.empty((M, N), dtype=torch.bfloat16, device=device),
                "ws": torch.empty((max(self.ws_bytes, 16),), dtype=torch.uint8, device=device),
                "q": torch.empty((M, K), dtype=torch.int8, device=device),
                "s_a": torch.empty((M,), dtype=torch.float32, device=device),
                "q2": torch.empty((M, K), dtype=torch.int8, device=device),
                "s_a2": torch.empty((M,), dtype=torch.float32, device=device),
            })
        self.x_host_bits = x_bits
        self.i = 0
        plan = w8a8.select(M, N, K)
        self.variant = plan["variant_name"]
        # the GEMV at 1-2 rows: quantization in its prologue (one launch);
        # otherwise the quantization kernel, then the GEMV or GEMM
        self.one_launch = self.variant == "gemv" and plan["quant_in_gemm_launch"] == 1
        self.launches_per_step = 1 if self.one_launch else 2

    def step(self):
        s = self.sets[self.i]
        self.i = (self.i + 1) % len(self.sets)
        self.w8a8.linear_fused(s["x"], s["Wq"], s["s_w"], s["b"], out=s["y"], workspace=s["ws"])

    def prepare_gemm_only(self):
        for s in self.sets:
            q, s_a = self.w8a8.quant_act(s["x"])
            s["q"].copy_(q)
            s["s_a"].copy_(s_a)
        torch.cuda.synchronize()

    def gemm_step(self):
        s = self.sets[self.i]
        self.i = (self.i + 1) % len(self.sets)
        self.w8a8.linear(s["q"], s["s_a"], s["Wq"], s["s_w"], s["b"], out=s["y"],
                         workspace=s["ws"])

    def quant_step(self):
        s = self.sets[self.i]
        self.i = (self.i + 1) % len(self.sets)
        B = self.w8a8.binding
        x = s["x"]
        st = B.w8a8_quant_act(B._ptr(x), x.shape[0], x.shape[1], x.stride(0), B._ptr(s["q2"]),
                              B._ptr(s["s_a2"]), B._stream())
        if st != 0:
            raise RuntimeError(B.status_string(st))


def timed(fn, steps: int, warmup: int, dist=None, sampler=None, graph=False, replays=1):
    """Run fn warmup times, then time `steps` calls with CUDA events on the
    current stream, bracketed by barrier + synchronize.  Returns seconds (max
    over ranks).  graph=True captures the `steps` calls into one CUDA graph
    first and times its replay (for layers shorter than their host-side
    launch cost); `replays` > 1 times that many back-to-back replays (the
    seconds returned are then for replays x steps calls)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if graph:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for _ in range(steps):
                    fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g.replay()                      # one untimed replay
        torch.cuda.synchronize()
        fn = g.replay
        steps_run = max(1, replays)
    else:
        steps_run = steps
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        # a ~0.1 ms spin ahead of the start event keeps the device busy while
        # the host enqueues the first steps, so the timed region holds the K
        # steps back to back and not the host's latency to the first launch
        torch.cuda._sleep(200_000)
        e0.record(stream)
        for _ in range(steps_run):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t = e0.elapsed_time(e1) / 1e3
    return max_over_ranks(t, dist)


def max_over_ranks(seconds: float, dist=None, device="cuda") -> float:
    """The slowest rank's time (every rank gets it): the job's time."""
    if dist is None:
        return seconds
    tt = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_rate(units_per_step_per_rank: float, steps: int, seconds: float, world: int) -> float:
    """Whole-job throughput of `world` replicas: the units all ranks processed
    over the (max-over-ranks) time."""
    return world * units_per_step_per_rank * steps / seconds


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def e2e_measure(layer: Layer, steps: int, warmup: int, dist=None):
    """The same layer through the C ABI call that takes HOST buffers: every
    step copies x from pinned host memory, runs the layer and copies y back."""
    w8a8 = layer.w8a8
    c = layer.case
    M, K, N = c.M, c.K, c.N
    dev = torch.device("cuda")
    x_host = torch.from_numpy(layer.x_host_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    s = layer.sets[0]
    x_dev = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    y_dev = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def fn():
        w8a8.linear_fused_host(x_host, s["Wq"], s["s_w"], s["b"], y_host, x_dev, y_dev, s["ws"])

    t = timed(fn, steps, warmup, dist)
    return t, 2 * M * K, 2 * M * N


def cpu_baseline(case: synth.LayerCase, budget_s: float = 12.0, max_rows: int = None):
    """The oracle, as it stands, on a bounded row sample of the workload:
    quantize the sampled rows, exact int32 GEMM against all N rows of Wq,
    fp32 epilogue.  Rows are sized from a calibration run to ~budget_s."""
    import oracle
    M, K, N = case.M, case.K, case.N
    x = case.x()
    wq, sw = oracle.quantize_weights(case.w())
    b = case.b()
    # calibrate on one row per oracle thread (it parallelizes over rows)
    rows = int(max(4, min(M, oracle.threads())))
    t0 = time.perf_counter()
    oracle.linear(x[:rows], wq, sw, b)
    dt = time.perf_counter() - t0
    rows = int(max(4, min(M, budget_s / max(dt, 1e-6) * rows)))
    if max_rows:
        rows = min(rows, max_rows)
    t0 = time.perf_counter()
    oracle.linear(x[:rows], wq, sw, b)
    dt = time.perf_counter() - t0
    return {"value": 2.0 * rows * N * K / dt / 1e12, "unit": "TOPS", "cores": oracle.threads(),
            "nproc": os.cpu_count(), "cpu_model": cpu_model(),
            "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"first {rows} of {M} rows of the {case.name} layer (all {N} outputs per row): "
                      f"per-token quant + exact int32 GEMM + fp32 epilogue, plain C with OpenMP"}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def single_launch_us(fn, reps: int = 20) -> float:
    """Median time of one isolated call: synchronize, then events around the
    call alone (the device idle before it)."""
    times = []
    for _ in range(reps):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    return statistics.median(times)


METRIC = "W8A8 linear int8 TOPS & % of tensor peak (quant+GEMM); M=1 GEMV HBM GB/s"
DTYPE = "int8 (int32 accumulate, fp32 epilogue, bf16 in/out)"
L2_NOTE = "inputs rotate over independent buffer sets totalling > 2x the 126 MB L2"


def workload_config(case: synth.LayerCase) -> dict:
    """The `config` of the JSON line: the workload alone, identical for both
    arms (no rank count, device or kernel choice in it)."""
    return {"workload": f"{case.name}: x bf16 [{case.M},{case.K}] ({case.x_kind}) @ Wq int8 "
                        f"[{case.N},{case.K}] + bias -> y bf16",
            "M": case.M, "K": case.K, "N": case.N, "seed": case.seed,
            "parallelism": "replicas (one independent layer call per GPU, no collective)",
            "l2": L2_NOTE}


def init_dist(world: int, local: int):
    """One process per GPU over NCCL, for the barrier around the timed region
    and the max-over-ranks reduction of the time."""
    if world <= 1:
        return None
    import torch.distributed as tdist
    from datetime import timedelta
    tdist.init_process_group("nccl", timeout=timedelta(seconds=120),
                             device_id=torch.device("cuda", local))
    return tdist


def build_line(args, m: dict, world: int) -> dict:
    """The JSON line of our arm from the measurements `m` (times already the
    max over ranks).  `value` is the whole job's rate: the operations of all
    `world` replicas over the slowest rank's time."""
    value = job_rate(m["ops_per_step"], args.steps, m["seconds"], world) / 1e12
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": m["warmup"],
        "ms_per_step": round(m["seconds"] / args.steps * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE, "data": "synthetic", "impl": "ours",
        "config": m["config"],
        "roofline": m.get("roofline"),
        "cpu_baseline": m.get("cpu_baseline"),
        "e2e": m.get("e2e"),
        "gpu_launches": m["launches_per_step"] * args.steps,
        "clocks": m.get("clocks"),
        "run": m.get("run"),
        "extras": m.get("extras"),
        "components": m.get("components", {}),
    }
    return line


def measure_i8_peak(dev, dist=None, iters: int = 2000, reps: int = 8) -> dict:
    """The device's dense int8 tensor-core rate, measured now as a burst:
    every CTA pair issues the GEMM's own tcgen05 kind::i8 instruction
    (M = N = 256, K = 32) from shared-memory operands, no global traffic;
    launches of ~0.6 ms, each timed alone, the fastest kept.  Called before
    any sustained load: under the 1 kW power cap a seconds-long loop settles
    at a lower clock (reported separately for the GEMM)."""
    import w8a8_int8_dynamic_token_b200 as w8a8
    B = w8a8.binding
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    pairs = sms // 2
    sampler = ClockSampler(dev.index if dev.index is not None else 0, period_s=0.0005)
    B.bench_mma_i8_peak(iters, pairs)
    torch.cuda.synchronize()
    best = float("inf")
    with sampler:
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            B.bench_mma_i8_peak(iters, pairs)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1) / 1e3)
    t = max_over_ranks(best, dist)
    status = w8a8.last_device_error()
    if status != 0:
        raise RuntimeError(f"peak loop: {w8a8.status_string(status)}")
    ops = pairs * iters * B.PEAK_OPS_PER_PAIR_ITERATION
    clk = sampler.summary()
    res = {"tops": round(ops / t / 1e12, 1), "us_per_launch": round(t * 1e6, 1),
           "pairs": pairs, "sm_mhz": clk.get("sm_mhz"), "clock_reasons": clk.get("reasons"),
           "timing": f"fastest of {reps} launches of {iters} iterations, each timed alone"}
    if clk.get("sm_mhz"):
        res["ops_per_clk_per_sm"] = round(ops / t / (clk["sm_mhz"] * 1e6) / (2 * pairs), 1)
    return res


def measure_int_mm(dev, dist=None, n: int = 8192, reps: int = 20) -> dict:
    """Library reference point: torch._int_mm (cuBLASLt int8 GEMM) at n^3,
    operands resident, the same int8 operation count convention; beside it
    this library's GEMM on the same operands (raw int32 output, as _int_mm
    returns) and with the bf16 epilogue, timed the same way."""
    import w8a8_int8_dynamic_token_b200 as w8a8
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    bt = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    b = bt.t()
    try:
        torch._int_mm(a, b)
    except Exception as e:  # not available in this build: say so
        return {"error": str(e)[:200]}
    ops = 2.0 * n ** 3
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    t = timed(lambda: torch._int_mm(a, b), reps, 3, dist, sampler) / reps
    ones = torch.ones(n, device=dev)
    acc = torch.empty((n, n), dtype=torch.int32, device=dev)
    y = torch.empty((n, n), dtype=torch.bfloat16, device=dev)
    B = w8a8.binding
    ws = torch.empty((w8a8.workspace_size(n, n, n),), dtype=torch.uint8, device=dev)

    def ours_raw():
        st = B.w8a8_linear(B._ptr(a), B._ptr(ones), n, n, B._ptr(bt), B._ptr(ones), None, n,
                           None, n, B._ptr(acc), B._ptr(ws), ws.numel(), B._stream())
        if st != 0:
            raise RuntimeError(B.status_string(st))

    def ours_bf16():
        st = B.w8a8_linear(B._ptr(a), B._ptr(ones), n, n, B._ptr(bt), B._ptr(ones), None, n,
                           B._ptr(y), n, None, B._ptr(ws), ws.numel(), B._stream())
        if st != 0:
            raise RuntimeError(B.status_string(st))

    t_raw = timed(ours_raw, reps, 3, dist) / reps
    t_bf16 = timed(ours_bf16, reps, 3, dist) / reps
    del a, b, bt, acc, y, ws
    torch.cuda.empty_cache()
    return {"tops": round(ops / t / 1e12, 1), "us": round(t * 1e6, 1), "n": n,
            "sm_mhz": sampler.summary().get("sm_mhz"),
            "ours_int32_out_tops": round(ops / t_raw / 1e12, 1),
            "ours_bf16_out_tops": round(ops / t_bf16 / 1e12, 1)}


def run_ours(args):
    rank, world, local = env_rank()
    torch.cuda.set_device(local if world > 1 else 0)
    dist = init_dist(world, local)
    dev = torch.device("cuda", torch.cuda.current_device())
    import w8a8_int8_dynamic_token_b200 as w8a8
    w8a8.lib()
    peaks = load_peaks()
    case = WORKLOADS[args.workload]
    M, K, N = case.M, case.K, case.N
    ops = 2.0 * M * N * K
    warmup = max(3, args.warmup)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    layer = Layer(case, dev)
    # few rows: the weight stream from HBM bounds the layer (GEMV or the
    # tensor-core small-M variant), and host launch cost is a large share of
    # it, so the steps are timed as a CUDA graph
    small = layer.variant in ("gemv", "gemv_tc")
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    t = timed(layer.step, args.steps, warmup, dist, sampler, graph=small)
    status = w8a8.last_device_error()
    if status != 0:
        raise RuntimeError(f"device error after the timed region: {w8a8.status_string(status)}")
    sec_per_step = t / args.steps

    # the same layer with the host launch cost removed (CUDA graph of the steps)
    layer.i = 0
    t_graph = timed(layer.step, args.steps, warmup, dist, graph=True) / args.steps
    # each kernel alone (q precomputed for the GEMM), same rotation, CUDA graphs
    layer.prepare_gemm_only()
    layer.i = 0
    gsteps = max(args.steps, 50)
    gsampler = ClockSampler(dev.index if dev.index is not None else 0)
    tg = timed(layer.gemm_step, gsteps, warmup, dist, gsampler, graph=True) / gsteps
    gclk = gsampler.summary()
    layer.i = 0
    tq = timed(layer.quant_step, gsteps, warmup, dist, graph=True) / gsteps
    if not small:
        # the burst peaks (the sustained GEMM run, which heats the part into
        # the power cap, comes last of all)
        i8 = measure_i8_peak(dev, dist)
        int_mm = measure_int_mm(dev, dist) if world == 1 else None
    if small:
        if layer.one_launch:
            # the GEMV quantizing its rows itself: the kernel is the layer
            algo_bytes = 2 * M * K + N * K + 6 * N + 2 * M * N
            t_kernel = sec_per_step
            kname, what = "gemv_i8", "gemv_i8 (fused quantization prologue)"
        else:
            # the kernel after the quantization kernel, reading q and s_a
            algo_bytes = M * K + 4 * M + N * K + 6 * N + 2 * M * N
            t_kernel = tg
            kname = "gemv_i8" if layer.variant == "gemv" else "gemm_i8_swapab"
            what = f"{kname} ({layer.variant}, after the quantization kernel)"
        achieved = algo_bytes / t_kernel / 1e9
        traffic, _ = profile_traffic(f"{kname}_{case.name}")
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": traffic, "kernel": what,
                    "peak_basis": f"{peaks['source']} HBM copy bandwidth (MEASURED_PEAKS.json)",
                    "algorithmic_bytes_per_launch": algo_bytes,
                    "us_per_launch": round(t_kernel * 1e6, 2),
                    "layer_frac_hbm": round((2 * M * K + N * K + 6 * N + 2 * M * N) / sec_per_step
                                            / 1e9 / peaks["hbm_gbs"], 4),
                    "timing": "CUDA graph of back-to-back calls"}
    else:
        derived = peaks["bf16_tflops"] * (NOMINAL_INT8_TOPS / NOMINAL_BF16_TFLOPS)
        achieved = ops / tg / 1e12
        traffic, _ = profile_traffic(f"gemm_i8_tcgen05_{case.name}")
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": i8["tops"],
                    "unit": "TFLOP/s", "frac": round(achieved / i8["tops"], 4),
                    "traffic": traffic,
                    "kernel": f"gemm_i8_tcgen05 ({layer.variant})",
                    "peak_basis": ("measured in this run: the tcgen05 kind::i8 M=256 N=256 K=32 "
                                   f"issue loop on all {i8['pairs']} CTA pairs, no memory traffic "
                                   "(int8 ops counted as TOPS)"),
                    "peak_measured_i8": i8,
                    "peak_bf16_x2": round(derived, 1),
                    "frac_of_peak_bf16_x2": round(achieved / derived, 4),
                    "peak_bf16_x2_basis": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s "
                                          "(MEASURED_PEAKS.json) x nominal int8/bf16 ratio 2",
                    "frac_of_nominal_4500": round(achieved / NOMINAL_INT8_TOPS, 4),
                    "us_per_launch": round(tg * 1e6, 2),
                    "sm_mhz_during_gemm": gclk.get("sm_mhz")}
        if int_mm is not None:
            roofline["torch_int_mm_8192"] = int_mm
            if int_mm.get("tops"):
                roofline["frac_of_torch_int_mm_8192"] = round(achieved / int_mm["tops"], 4)
    quant_bytes = 3 * M * K + 4 * M
    layer.i = 0
    t_single = single_launch_us(layer.step)
    extras = {
        "layer_us": round(sec_per_step * 1e6, 2),
        "layer_single_call_us": round(t_single, 2),
        "layer_us_graph": round(t_graph * 1e6, 2),
        "layer_tops_graph": round(ops / t_graph / 1e12, 1),
        "layer_frac_of_nominal_4500": round(ops / sec_per_step / 1e12 / NOMINAL_INT8_TOPS, 4),
        "gemm_us": round(tg * 1e6, 2),
        "quant_us": round(tq * 1e6, 2),
        "quant_gbs": round(quant_bytes / tq / 1e9, 1),
        "quant_frac_hbm": round(quant_bytes / tq / 1e9 / peaks["hbm_gbs"], 4),
    }

    e2e = None
    if not args.no_e2e:
        esteps = max(3, min(args.steps, 20))
        te, h2d, d2h = e2e_measure(layer, esteps, 2, dist)
        e2e = {"value": round(job_rate(ops, esteps, te, world) / 1e12, 3), "unit": "TOPS",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(te / esteps * 1e3, 3)}
    launches = layer.launches_per_step

    components = {}
    if not args.no_extras and world == 1:
        components = extra_components(args, dev, dist, peaks, world,
                                      roofline.get("peak") if not small else None)

    if not small:
        # the SM clock the GEMM holds under sustained load (the power cap can
        # hold it below the clock of a short burst): about 0.4 s of graph
        # replays of the same GEMM steps, sampled every 2 ms -- run last, so
        # that the heat it leaves throttles no other measurement
        layer.i = 0
        lsampler = ClockSampler(dev.index if dev.index is not None else 0)
        reps = max(2, int(0.4 / max(tg * gsteps, 1e-6)))
        tl = timed(layer.gemm_step, gsteps, 0, dist, lsampler, graph=True, replays=reps)
        gload = dict(lsampler.summary(), us_per_launch=round(tl / (reps * gsteps) * 1e6, 2),
                     seconds=round(tl, 3))
        roofline["gemm_sustained_0p4s"] = gload
        if gload.get("sm_mhz") and i8.get("ops_per_clk_per_sm"):
            # the measured per-clock rate at the clock the GEMM holds under
            # sustained load, against the GEMM's rate in that same run
            clock_peak = sms * i8["ops_per_clk_per_sm"] * gload["sm_mhz"] * 1e6 / 1e12
            sustained = ops / (gload["us_per_launch"] * 1e-6) / 1e12
            roofline["frac_of_peak_at_gemm_clock"] = round(sustained / clock_peak, 4)
            roofline["peak_at_gemm_clock_tops"] = round(clock_peak, 1)
            roofline["gemm_clock_basis"] = ("median SM clock of the 0.4 s sustained run; its "
                                            "rate against the measured per-clock peak")
    del layer
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(case, budget_s=args.cpu_budget)

    if dist is not None:
        dist.barrier()
    m = {"seconds": t, "ops_per_step": ops, "warmup": warmup, "config": workload_config(case),
         "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "launches_per_step": launches,
         "clocks": sampler.summary(), "extras": extras, "components": components,
         "run": {"gpu": torch.cuda.get_device_name(dev), "sms": sms,
                 "kernel_variant": layer_variant_name(case), "ranks": world}}
    if rank == 0:
        print(json.dumps(build_line(args, m, world)), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def layer_variant_name(case):
    import w8a8_int8_dynamic_token_b200 as w8a8
    return w8a8.select(case.M, case.N, case.K)["variant_name"]


def extra_components(args, dev, dist, peaks, world, i8_peak=None):
    """The other workloads of the same metric: the M = 1 / 2 AdaLN GEMV (HBM
    GB/s), the FFN up/down pair, each layer alone and back to back, one DiT
    block, the small-M regime, the M sweep over the block's linear shapes,
    packed-weight loading and the W8A16 variant."""
    out = {}
    steps = max(20, min(args.steps, 200))
    for case in (synth.ADALN_M1, synth.ADALN_M2, synth.ADALN_M16):
        L = Layer(case, dev)
        t = timed(L.step, steps * 5, 5, dist, graph=True) / (steps * 5)
        t_eager = timed(L.step, steps * 5, 5, dist) / (steps * 5)
        M, K, N = case.M, case.K, case.N
        algo_bytes = 2 * M * K + N * K + 4 * N + 2 * N + 2 * M * N
        gbs = algo_bytes / t / 1e9
        out[case.name] = {"us": round(t * 1e6, 2), "GBs": round(gbs, 1),
                          "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                          "TOPS": round(2 * M * N * K / t / 1e12, 3), "variant": L.variant,
                          "us_eager_launches": round(t_eager * 1e6, 2), "timing": "CUDA graph of back-to-back calls",
                          "sets_rotated": len(L.sets)}
        del L
        torch.cuda.empty_cache()
    if args.workload == "qkv":
        layers = {}
        for case in (synth.FFN_UP, synth.FFN_DOWN):
            L = Layer(case, dev)
            t = timed(L.step, steps, 5, dist) / steps
            ops = 2 * case.M * case.N * case.K
            out[case.name] = {"us": round(t * 1e6, 2), "TOPS": round(ops / t / 1e12, 1),
                              "frac_of_nominal_4500": round(ops / t / 1e12 / NOMINAL_INT8_TOPS, 4),
                              "variant": L.variant}
            out[case.name].update(layer_breakdown(L, steps, dist, peaks))
            L.i = 0
            layers[case.name] = L
        up, down = layers["ffn_up"], layers["ffn_down"]

        def pair():
            up.step()
            down.step()

        t = timed(pair, steps, 5, dist) / steps
        ops = 2 * up.case.M * up.case.N * up.case.K + 2 * down.case.M * down.case.N * down.case.K
        out["ffn_pair"] = {"us": round(t * 1e6, 2), "TOPS": round(ops / t / 1e12, 1),
                           "frac_of_nominal_4500": round(ops / t / 1e12 / NOMINAL_INT8_TOPS, 4)}
        del layers, up, down
        torch.cuda.empty_cache()
        out["dit_block"] = dit_block_component(dev, dist, max(10, steps // 4))
        out["small_m"] = small_m_component(dev, dist, peaks, steps)
        if not args.no_sweep:
            out["sweep"] = sweep_component(dev, dist, peaks, i8_peak)
        out["unpack_int32_weights"] = unpack_component(dev, dist, peaks, steps)
        out["w8a16_qkv"] = w8a16_component(dev, dist, peaks, steps)
    return out


def layer_breakdown(L, steps, dist, peaks) -> dict:
    """The layer's two kernels timed alone (CUDA graphs, same rotation): the
    GEMM on precomputed q and the per-token quantization."""
    M, K = L.case.M, L.case.K
    L.prepare_gemm_only()
    L.i = 0
    tg = timed(L.gemm_step, steps, 3, dist, graph=True) / steps
    L.i = 0
    tq = timed(L.quant_step, steps, 3, dist, graph=True) / steps
    qbytes = 3 * M * K + 4 * M
    return {"gemm_us": round(tg * 1e6, 2), "gemm_TOPS": round(L.case.ops / tg / 1e12, 1),
            "quant_us": round(tq * 1e6, 2), "quant_GBs": round(qbytes / tq / 1e9, 1),
            "quant_frac_hbm": round(qbytes / tq / 1e9 / peaks["hbm_gbs"], 4)}


def w8a16_component(dev, dist, peaks, steps):
    """The weight-only variant on the QKV shape: bf16 x [4352, 3072] against
    int8 Wq [9216, 3072] widened to bf16 in the kernel, bf16 tensor cores."""
    import w8a8_int8_dynamic_token_b200 as w8a8
    case = synth.QKV
    M, K, N = case.M, case.K, case.N
    W = bf16_dev(case.w(), dev)
    Wq, s_w = w8a8.quantize_weights(W)
    del W
    x0 = bf16_dev(case.x(), dev)
    nsets = n_sets(2 * M * K + N * K + 2 * M * N)
    sets = [(x0.clone(), Wq.clone(), torch.empty((M, N), dtype=torch.bfloat16, device=dev))
            for _ in range(nsets)]
    i = [0]

    def step():
        x, wq, y = sets[i[0] % nsets]
        i[0] += 1
        w8a8.w8a16_linear(x, wq, s_w, out=y)

    t = timed(step, steps, 5, dist, graph=True) / steps
    tflops = case.ops / t / 1e12
    del sets
    torch.cuda.empty_cache()
    return {"us": round(t * 1e6, 2), "TFLOPS": round(tflops, 1),
            "frac_of_bf16_peak": round(tflops / peaks["bf16_tflops"], 4),
            "peak_basis": "measured bf16 burst (MEASURED_PEAKS.json)"}


def sweep_component(dev, dist, peaks, i8_peak, oracle_rows: int = 4):
    """The M sweep over one DiT block's linear shapes: M in {1, 16, 17, 256,
    1024, 4352, 8704, 16384} x (K, N) in {(3072, 9216), (3072, 3072),
    (3072, 12288), (12288, 3072)}, seed 0 (seeds 1-3 are parity cases).  Per
    point: the whole layer (quantization included) in a CUDA graph of
    back-to-back calls with inputs rotated over > 2x L2, its TOPS, the
    algorithmic GB/s, and the fraction of the attainable rate
    min(peak_i8, AI * HBM) with AI = 2MNK / (2MK + NK + 6N + 2MN); and the
    oracle's rate on a few rows of the same layer (plain C, all host cores)."""
    import oracle
    points = []
    bw = peaks["hbm_gbs"] * 1e9
    for K, N in synth.SWEEP_KN:
        kind = "gelu" if K == 12288 else "studentt"
        w_bits = synth.make_w(N, K, 0)
        weights = quantized_weights(w_bits, dev)
        wq_h, sw_h = oracle.quantize_weights(w_bits)
        for M in synth.SWEEP_M:
            case = synth.LayerCase(f"sweep_m{M}_k{K}_n{N}_s0", M, K, N, kind, 0)
            x_bits = case.x()
            L = Layer(case, dev, x_bits=x_bits, weights=weights)
            ops = 2.0 * M * N * K
            steps = int(min(200, max(10, 2e-2 / max(ops / 3e15, 2e-6))))   # ~20 ms of work
            t = timed(L.step, steps, 3, dist, graph=True) / steps
            algo = 2 * M * K + N * K + 6 * N + 2 * M * N
            ai = ops / algo
            peak_ops = i8_peak * 1e12 if i8_peak else NOMINAL_INT8_TOPS * 1e12
            attain = min(peak_ops, ai * bw)
            rows = min(M, oracle_rows)
            t0 = time.perf_counter()
            oracle.linear(x_bits[:rows], wq_h, sw_h, case.b())
            t_or = time.perf_counter() - t0
            points.append({"M": M, "K": K, "N": N, "variant": L.variant, "us": round(t * 1e6, 2),
                           "TOPS": round(ops / t / 1e12, 1), "GBs": round(algo / t / 1e9, 1),
                           "bound": "hbm" if ai * bw < peak_ops else "tensor",
                           "frac_of_attainable": round(ops / t / attain, 4),
                           "frac_of_nominal_4500": round(ops / t / 1e12 / NOMINAL_INT8_TOPS, 4),
                           "oracle_TOPS": round(2.0 * rows * N * K / t_or / 1e12, 5),
                           "oracle_rows": rows})
            del L
            torch.cuda.empty_cache()
        del weights
        torch.cuda.empty_cache()
    return {"points": points,
            "attainable": "min(measured int8 peak of this run, AI x measured HBM GB/s)",
            "timing": "CUDA graph of back-to-back layer calls (quantization + GEMM or the GEMV), "
                      "inputs rotated over > 2x L2; seed 0",
            "oracle": f"CPU oracle on the first {oracle_rows} rows of each layer, all outputs"}


def quantized_weights(w_bits, dev):
    """Quantize a host bf16 weight once on the device, for several layers."""
    import w8a8_int8_dynamic_token_b200 as w8a8
    W = bf16_dev(w_bits, dev)
    Wq, s_w = w8a8.quantize_weights(W)
    del W
    return Wq, s_w


def small_m_component(dev, dist, peaks, steps):
    """The selector's small-M regime on the QKV weight (K = 3072, N = 9216):
    whole layer per M, with the kernel chosen, TOPS and the weight-stream
    bandwidth (these layers are bound by reading Wq once)."""
    res = {}
    for M in (16, 17, 64, 128, 256, 512, 1024):
        case = synth.LayerCase(f"qkv_m{M}", M, 3072, 9216, "studentt", 0)
        L = Layer(case, dev)
        t = timed(L.step, steps, 5, dist, graph=True) / steps
        algo = 2 * M * case.K + case.N * case.K + 6 * case.N + 2 * M * case.N
        res[f"M={M}"] = {"us": round(t * 1e6, 2), "variant": L.variant,
                         "TOPS": round(case.ops / t / 1e12, 1),
                         "GBs": round(algo / t / 1e9, 1),
                         "frac_hbm": round(algo / t / 1e9 / peaks["hbm_gbs"], 4)}
        del L
        torch.cuda.empty_cache()
    res["timing"] = "CUDA graph of back-to-back layer calls, inputs rotated over > 2x L2"
    return res


def unpack_component(dev, dist, peaks, steps):
    """Loading packed int32 weight storage (four codes biased by 128 per word)
    into the GEMM's int8 layout: the AdaLN weight, 18432 x 3072."""
    import w8a8_int8_dynamic_token_b200 as w8a8
    N, K = 18432, 3072
    nsets = n_sets(2 * N * K)
    packed = [torch.randint(-2**31, 2**31 - 1, (N, K // 4), dtype=torch.int32, device=dev)
              for _ in range(nsets)]
    outs = [torch.empty((N, K), dtype=torch.int8, device=dev) for _ in range(nsets)]
    B = w8a8.binding
    i = [0]

    def step():
        j = i[0] % nsets
        i[0] += 1
        st = B.w8a8_unpack_int32_weights(B._ptr(packed[j]), N, K, B._ptr(outs[j]), B._stream())
        if st != 0:
            raise RuntimeError(B.status_string(st))

    t = timed(step, steps, 5, dist, graph=True) / steps
    gbs = 2 * N * K / t / 1e9
    del packed, outs
    torch.cuda.empty_cache()
    return {"us": round(t * 1e6, 2), "GBs": round(gbs, 1),
            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "bytes_per_launch": 2 * N * K}


def dit_block_component(dev, dist, steps):
    """One DiT block's quantized linears at CFG batch 2, launched back to back
    on one stream (each call's kernels are programmatic dependents of the
    previous call's): eager launches and a CUDA graph of the block."""
    layers = [Layer(c, dev) for c in synth.DIT_BLOCK]

    def block():
        for L in layers:
            L.step()

    t = timed(block, steps, 3, dist) / steps
    for L in layers:
        L.i = 0
    t_graph = timed(block, steps, 3, dist, graph=True) / steps
    per_layer = {}
    for L in layers:
        L.i = 0
        us = round(timed(L.step, steps, 3, dist, graph=True) / steps * 1e6, 2)
        per_layer[L.case.name] = {"us": us, "frac_of_nominal_4500":
                                  round(L.case.ops / us / 1e6 / NOMINAL_INT8_TOPS, 4)}
    ops = sum(c.ops for c in synth.DIT_BLOCK)
    res = {"us": round(t * 1e6, 2), "TOPS": round(ops / t / 1e12, 1),
           "us_graph": round(t_graph * 1e6, 2), "TOPS_graph": round(ops / t_graph / 1e12, 1),
           "frac_of_nominal_4500_graph": round(ops / t_graph / 1e12 / NOMINAL_INT8_TOPS, 4),
           "layers_us_graph_alone": per_layer,
           "calls": [f"{c.name} M={c.M} K={c.K} N={c.N}" for c in synth.DIT_BLOCK],
           "gpu_launches_per_block": sum(L.launches_per_step for L in layers)}
    del layers
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return
    import oracle
    case = WORKLOADS[args.workload]
    M, K, N = case.M, case.K, case.N
    x = case.x()
    wq, sw = oracle.quantize_weights(case.w())
    b = case.b()
    # rows per step so the whole run (warmup + steps) takes a few minutes at most
    t0 = time.perf_counter()
    oracle.linear(x[:2], wq, sw, b)
    per_row = (time.perf_counter() - t0) / 2
    total_steps = max(1, args.steps) + max(3, args.warmup)
    rows = int(max(1, min(M, 90.0 / total_steps / max(per_row, 1e-9))))
    for i in range(max(3, args.warmup)):
        oracle.linear(x[:rows], wq, sw, b)
    times = []
    for i in range(max(1, args.steps)):
        r0 = (i * rows) % max(1, M - rows + 1)
        t0 = time.perf_counter()
        oracle.linear(x[r0:r0 + rows], wq, sw, b)
        times.append(time.perf_counter() - t0)
    t = sum(times)
    value = 2.0 * rows * N * K * len(times) / t / 1e12
    sample = (f"{rows} of {M} rows of the {case.name} layer per step (all {N} outputs per row): "
              f"per-token quant + exact int32 GEMM + fp32 epilogue, plain C with OpenMP")
    line = {
        "metric": METRIC,
        "value": round(value, 6), "unit": "TOPS", "n_gpus": world, "steps": len(times),
        "warmup": max(3, args.warmup), "ms_per_step": round(t / len(times) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE, "data": "synthetic",
        "impl": "reference",
        "config": workload_config(case),
        "run": {"ranks": world, "oracle_on": "rank 0 only"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def launcher_argv(n: int, port: int, argv=None) -> list:
    """The torchrun command that runs this script as n ranks on this node,
    one per GPU, rendezvous on 127.0.0.1."""
    argv = sys.argv[1:] if argv is None else argv
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def relaunch_under_torchrun(n: int):
    """`--gpus N` without a launcher: replace this process by torchrun with N
    ranks (each rank then sees WORLD_SIZE and runs its replica)."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    sys.stdout.flush()
    cmd = launcher_argv(n, port)
    os.execv(cmd[0], cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="qkv")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-sweep", action="store_true")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        relaunch_under_torchrun(args.gpus)   # does not return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
