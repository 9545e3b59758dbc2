#!/usr/bin/env python3
"""Benchmark of the fused tensor-core GEMM (libtlgemm.so) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one C = epilogue(A . B) call through the C ABI on the workload's
full size.  The default workload is the largest configuration: a transformer
MLP up-projection, 8192 x 16384 x 4096 in bf16 with the fused bias + exact
GELU epilogue (the fused epilogue is what the TileLang GPU kernel design
article, paragraph 5, is about).  Inputs are seeded synthetic data, resident
in HBM before the timed region; the timed region rotates over enough
input/output sets that every step reads operands that are not in L2.  Timing
uses CUDA events on the launching stream; with N > 1 (torchrun, one process
per GPU) each rank runs an independent replica (weak scaling, no data-path
collective) and the slowest rank's time counts.

Beside the headline the JSON line carries:
  per_config  every GEMM configuration of the benchmark set (the pages' 4096^3
              fp16 GEMM with and without the epilogue, the small fused case,
              the MLP up-projection, and the ragged / tall / skinny bf16
              shapes with and without bias + GELU), each timed the same way
              as a short burst: TFLOP/s, the fraction of the measured dense
              peak, GB/s of compulsory traffic and its fraction of the
              measured HBM copy bandwidth, and the same GEMM with its operands
              left warm in L2;
  sustained   the headline GEMM run back to back for a few seconds, in the
              power-capped steady state, against the sustained peak.
A timed region shorter than a second is a burst and is compared with the
burst peak; a longer one with the sustained peak.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle
instead (the same bounded row samples of the same workload on the host cores
that the cpu_baseline figure uses).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = ("GEMM TFLOP/s (1×B200) and fraction of dense fp16/bf16 tensor peak, ±bias+GELU")
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# A timed region at least this long runs in the power-capped steady state.
SUSTAINED_REGION_S = 1.0
# Multiply-adds of one oracle call (one sample): about 2 s on 16 host cores.
ORACLE_SAMPLE_MACS = 1 << 35

# The benchmark set: every GEMM configuration the metric is quoted on.
PER_CONFIG = (
    "gemm256_f16_bias_gelu",
    "gemm4096_f16",
    "gemm4096_f16_bias_gelu",
    "mlp_up_8192x16384x4096_bf16_bias_gelu",
    "ragged_4000x3000x2050_bf16",
    "ragged_4000x3000x2050_bf16_bias_gelu",
    "tall_16384x1024x8192_bf16",
    "tall_16384x1024x8192_bf16_bias_gelu",
    "skinny_128x16384x4096_bf16",
    "skinny_128x16384x4096_bf16_bias_gelu",
)


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend, ws):
    import datetime
    import torch.distributed as dist
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if ws > 1 else None


def max_over_ranks(value: float, dist, device=None) -> float:
    """The largest `value` over all ranks (each rank passes its own)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / seconds_max


# ------------------------------------------------------------------ roofline inputs
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks: dict, region_s: float):
    """(peak TFLOP/s, its name) for a timed region of `region_s` seconds: a
    burst is compared with the burst figure, a region of a second or more
    with the sustained (power-capped) figure.  fp16 and bf16 share the dense
    tensor rate."""
    burst = float(peaks["bf16_tflops"])
    if region_s >= SUSTAINED_REGION_S:
        return float(peaks.get("bf16_tflops_sustained", burst)), "bf16_tflops_sustained"
    return burst, "bf16_tflops"


# Below this time at the roofline a GEMM is bound by launch latency.
LATENCY_BOUND_S = 5e-6


def bound_of(w) -> str:
    """What bounds the workload at the measured peaks: 'latency' when both its
    tensor time and its compulsory-traffic time are a few microseconds (the
    256^3 case), 'hbm' when the traffic takes longer than the flops (the
    skinny 128-row shape), else 'tensor'."""
    peaks, _ = measured_peaks()
    t_tensor = w.flops / (float(peaks["bf16_tflops"]) * 1e12)
    t_hbm = w.min_bytes() / (float(peaks["hbm_gbs"]) * 1e9)
    if max(t_tensor, t_hbm) < LATENCY_BOUND_S:
        return "latency"
    return "hbm" if t_hbm > t_tensor else "tensor"


# The files the GEMM kernel's code and launch are built from; a traffic figure
# taken on other sources of these files no longer describes the kernel.
GEMM_SOURCES = ("sm100.cuh", "gemm_kernel.cuh", "config_table.inc", "tl_gemm.cu")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tensor_core_gemm_tl_b200", "csrc")
    for name in GEMM_SOURCES:
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(name.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


_TRAFFIC_RE = re.compile(r"<!--\s*traffic\s+workload=(\S+)\s+src=(\S+)\s+bytes_per_launch=(\d+)\s*-->")


def ncu_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    src = kernel_source_hash()
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for m in _TRAFFIC_RE.finditer(open(f).read()):
            if m.group(1) == workload and m.group(2) == src:
                return int(m.group(3))
    return None


# ------------------------------------------------------------------ clocks during the timed region
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.0005):
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
        except Exception as e:  # NVML missing: report no clocks rather than guess
            log("clock sampling unavailable:", e)
            self.max_mhz = None
        self._stop = threading.Event()

    def _sample(self):
        nv = self.nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._sample()  # at least one sample even for a region shorter than the period
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ the oracle as a CPU baseline
def oracle_sample_rows(w, seed: int = 0) -> np.ndarray:
    """The rows of C one oracle sample computes: a fixed number of multiply-adds
    (ORACLE_SAMPLE_MACS), rows drawn without replacement, sorted."""
    n = int(max(1, min(w.M, round(ORACLE_SAMPLE_MACS / (w.N * w.K)))))
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(w.M, size=n, replace=False))


def oracle_sample(w, A, B, bias, rows):
    """One oracle call on `rows` rows of C: (seconds, flops)."""
    import oracle  # test infrastructure: the CPU-baseline leg and the reference arm only
    t0 = time.perf_counter()
    oracle.gemm(A, B, bias, w.dtype, w.epi, rows=rows)
    return time.perf_counter() - t0, 2.0 * len(rows) * w.N * w.K


def cpu_baseline(w, A, B, bias, budget_s=12.0):
    """Oracle throughput: samples of the same size as the reference arm's
    steps, as many as fit in about budget_s (at least one)."""
    import oracle
    rows = oracle_sample_rows(w)
    t_tot = f_tot = 0.0
    calls = 0
    while calls == 0 or t_tot + t_tot / calls <= budget_s:
        t, f = oracle_sample(w, A, B, bias, rows)
        t_tot += t
        f_tot += f
        calls += 1
    return {"value": f_tot / t_tot / 1e12, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{calls} oracle calls of {len(rows)} of {w.M} rows of C each "
                      f"({len(rows)}x{w.N}x{w.K} multiply-adds, fp64), {t_tot:.1f} s"}


# ------------------------------------------------------------------ the GPU arm
def ensure_library():
    """Build libtlgemm.so in-tree if it is missing (nvcc, sm_100a)."""
    import importlib.util
    path = os.path.join(ROOT, "tensor_core_gemm_tl_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_tl_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    if not os.path.exists(mod.LIB):
        mod.build(force=True)


def rotation_sets(w) -> int:
    """Input/output sets the timed region rotates over: together at least
    three times the L2, so every step's operands come from HBM."""
    set_bytes = 2 * (w.M * w.K + w.K * w.N + w.M * w.N)
    return max(2, int(np.ceil(3 * L2_BYTES / set_bytes)))


def l2_note(w) -> str:
    set_bytes = 2 * (w.M * w.K + w.K * w.N + w.M * w.N)
    n = rotation_sets(w)
    return (f"inputs larger than L2: {n} rotating input/output sets of {set_bytes / 2**20:.0f} MiB "
            f"({n * set_bytes / 2**20:.0f} MiB > {L2_BYTES / 2**20:.0f} MiB L2)")


def common_config(w, seed: int, ws: int) -> dict:
    """The workload keys both arms print."""
    return {**w.describe(), "seed": seed, "parallelism": f"replicas{ws}" if ws > 1 else "single",
            "l2": l2_note(w)}


class GemmBench:
    """Device buffers of one workload and the launch of one step."""

    _host_cache: dict = {}

    def __init__(self, w, dev, seed, tg):
        import torch
        self.w, self.dev, self.tg = w, dev, tg
        self.tdt = torch.float16 if w.dtype == wl.F16 else torch.bfloat16
        self.A_bits, self.B_bits, self.bias_bits = self.host_inputs(w, seed)

        def dev_tensor(bits):
            return torch.from_numpy(bits.view(np.int16)).to(dev).view(self.tdt)

        A0, B0 = dev_tensor(self.A_bits), dev_tensor(self.B_bits)
        self.bias = dev_tensor(self.bias_bits) if self.bias_bits is not None else None
        self.nsets = rotation_sets(w)
        self.sets = []
        for i in range(self.nsets):
            self.sets.append((A0 if i == 0 else A0.clone(), B0 if i == 0 else B0.clone(),
                              torch.empty((w.M, w.N), dtype=self.tdt, device=dev)))
        self.epi = "bias_gelu" if w.epi == wl.EPI_BIAS_GELU else None
        s0 = self.sets[0]
        self.plan = tg.plan(w.M, w.N, w.K, w.dtype, self.epi,
                            num_sms=torch.cuda.get_device_properties(dev).multi_processor_count,
                            ptrs=(s0[0].data_ptr(), s0[1].data_ptr(),
                                  self.bias.data_ptr() if self.bias is not None else 0, s0[2].data_ptr()))
        self.launches_per_step = 1 + self.plan["pad_a"] + self.plan["pad_b"]

    @classmethod
    def host_inputs(cls, w, seed):
        # the plain and the bias + GELU form of a shape draw the same A and B
        key = (w.M, w.N, w.K, w.dtype, w.a, w.b, seed)
        if key not in cls._host_cache:
            cls._host_cache.clear()
            A, B, _ = wl.make_inputs(wl.Workload(w.name, w.M, w.N, w.K, w.dtype, wl.EPI_NONE, w.a, w.b, None), seed)
            cls._host_cache[key] = (A, B)
        A, B = cls._host_cache[key]
        return A, B, wl.make_bias(w, seed)

    def step(self, i, stream, rotate=True):
        A, B, C = self.sets[i % self.nsets if rotate else 0]
        self.tg.gemm(A, B, self.bias, epilogue=self.epi, out=C, stream=stream)

    def free(self):
        self.sets = []
        self.bias = None


def timed_region(gb, stream, steps, warmup, ramp_s, rotate=True, sampler=None, dist=None):
    """Run an untimed clock ramp and `warmup` steps, then time exactly `steps`
    steps between two events on `stream` (barrier and synchronize on both
    sides).  Returns the region's milliseconds on this rank."""
    import torch
    t_end = time.time() + ramp_s
    i = 0
    while time.time() < t_end:
        for _ in range(5):
            gb.step(i, stream, rotate)
            i += 1
        torch.cuda.synchronize()
    for j in range(warmup):
        gb.step(j, stream, rotate)
    torch.cuda.synchronize()
    if gb.tg.check_device() != 0:
        raise RuntimeError(f"device error during the warm-up of {gb.w.name}")
    # Events only at the two ends of the region: an event between launches
    # would serialise them and hide the overlap of one kernel's set-up with the
    # previous kernel's tail.
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ctx = sampler if sampler is not None else _NullCtx()
    with ctx:
        t0.record(stream)
        for j in range(steps):
            gb.step(j, stream, rotate)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    if gb.tg.check_device() != 0:
        raise RuntimeError(f"device error in the timed region of {gb.w.name}")
    return t0.elapsed_time(t1)


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def per_config_entry(w, gb, ms, warm_ms, peaks, clocks):
    tflops = w.flops / (ms / 1e3) / 1e12
    gbs = w.min_bytes() / (ms / 1e3) / 1e9
    peak, peak_name = tensor_peak(peaks, 0.0)
    hbm = float(peaks["hbm_gbs"])
    bound = bound_of(w)
    e = {"ms": round(ms, 5), "tflops": round(tflops, 2), "frac": round(tflops / peak, 4),
         "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4), "bound": bound,
         "warm_l2_tflops": round(w.flops / (warm_ms / 1e3) / 1e12, 2),
         "kernel_config": gb.plan["config_name"], "split": gb.plan["split"],
         "raster_group": gb.plan["raster_group"],
         "launches_per_step": gb.launches_per_step, "sm_mhz": clocks["sm_mhz"],
         "reasons": clocks["reasons"]}
    # the roofline fraction of the bound that applies
    e["roofline_frac"] = e["frac_hbm"] if bound == "hbm" else e["frac"]
    return e


# The attention forward (the library's next kernel on the tensor cores): the
# shapes it is measured on, (batch, heads, seq, head_dim, causal), bf16.
ATTENTION_SHAPES = ((4, 16, 4096, 128, False), (4, 16, 4096, 128, True), (8, 16, 2048, 64, False),
                    (8, 16, 2048, 64, True))


def attention_entries(args, stream, peaks, dist, dev):
    """tl_attention_fwd timed like the GEMM bursts (a region of back-to-back
    launches after an idle pause), with PyTorch's scaled_dot_product_attention
    on the same inputs beside it as context."""
    import torch
    import torch.nn.functional as F
    import tensor_core_gemm_tl_b200 as tg
    from tensor_core_gemm_tl_b200.compare import attention_flops
    burst, _ = tensor_peak(peaks, 0.0)
    out = {}
    for B, H, S, D, causal in ATTENTION_SHAPES:
        g = torch.Generator(device=dev).manual_seed(0)
        q, k, v = (torch.randn(B, H, S, D, device=dev, dtype=torch.bfloat16, generator=g) for _ in range(3))
        o = torch.empty_like(q)
        fl = attention_flops(B, H, S, S, D, causal)

        def region(fn):
            time.sleep(args.rest_s)
            for _ in range(args.warmup):
                fn()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            if dist:
                dist.barrier()
            torch.cuda.synchronize()
            t0.record(stream)
            for _ in range(args.steps):
                fn()
            t1.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks(t0.elapsed_time(t1) / args.steps, dist, dev)

        ms = region(lambda: tg.attention(q, k, v, causal=causal, out=o, stream=stream))
        if tg.check_device() != 0:
            raise RuntimeError("device error in the attention region")
        ms_sdpa = region(lambda: F.scaled_dot_product_attention(q, k, v, is_causal=causal))
        tf, tf_sdpa = fl / (ms / 1e3) / 1e12, fl / (ms_sdpa / 1e3) / 1e12
        out[f"b{B}h{H}s{S}d{D}{'_causal' if causal else ''}_bf16"] = {
            "ms": round(ms, 5), "tflops": round(tf, 1), "frac": round(tf / burst, 4),
            "torch_sdpa_tflops": round(tf_sdpa, 1), "of_sdpa": round(tf / tf_sdpa, 3)}
        del q, k, v, o
    return out


def run_gpu(args, w):
    import torch
    ws, rank, local = dist_env()
    dist = init_dist("nccl", ws)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    ensure_library()
    import tensor_core_gemm_tl_b200 as tg

    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = measured_peaks()
    K = args.steps

    # ---------------------------------------------------------------- headline: a burst
    head = GemmBench(w, dev, args.seed, tg)
    sampler = ClockSampler(local)
    region_ms = timed_region(head, stream, K, args.warmup, args.ramp_s, sampler=sampler, dist=dist)
    region_ms_max = max_over_ranks(region_ms, dist, dev)
    clocks = sampler.summary()
    kernel_ms = region_ms / K  # one GEMM launch per step (plus the pad copies when an operand needs them)
    value = aggregate(w.flops * K, region_ms_max / 1e3, ws) / 1e12
    peak, peak_name = tensor_peak(peaks, region_ms_max / 1e3)
    achieved = w.flops / (kernel_ms / 1e3) / 1e12
    bound = bound_of(w)
    roof = {"bound": bound, "unit": UNIT, "traffic": ncu_traffic(w.name),
            "kernel_ms": round(kernel_ms, 5), "kernel_ms_is": "timed region / GEMM launches",
            "algorithmic_flops_per_launch": w.flops, "min_hbm_bytes_per_launch": w.min_bytes(),
            "region_s": round(region_ms_max / 1e3, 4)}
    if bound == "hbm":
        gbs = w.min_bytes() / (kernel_ms / 1e3) / 1e9
        roof.update({"achieved": round(gbs, 1), "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                     "frac": round(gbs / float(peaks["hbm_gbs"]), 4),
                     "peak_source": f"{peak_src} hbm_gbs (copy)", "tflops": round(achieved, 2)})
    else:
        roof.update({"achieved": round(achieved, 2), "peak": peak, "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_src} {peak_name} (cuBLAS; a region under "
                                    f"{SUSTAINED_REGION_S:g} s is a burst); fp16 dense rate equals bf16"})

    # ---------------------------------------------------------------- every configuration, as a burst
    per_config = {}
    if not args.no_per_config:
        for name in PER_CONFIG:
            wc = wl.WORKLOADS[name]
            b = head if name == w.name else GemmBench(wc, dev, args.seed, tg)
            # each region starts after an idle pause, so that it runs at the
            # unthrottled clock like the headline burst
            time.sleep(args.rest_s)
            cs = ClockSampler(local)
            ms = max_over_ranks(timed_region(b, stream, K, args.warmup, args.ramp_s, sampler=cs, dist=dist),
                                dist, dev) / K
            time.sleep(args.rest_s)
            warm_ms = max_over_ranks(timed_region(b, stream, K, args.warmup, args.ramp_s, rotate=False, dist=dist),
                                     dist, dev) / K
            per_config[name] = per_config_entry(wc, b, ms, warm_ms, peaks, cs.summary())
            if b is not head:
                b.free()
                del b
            torch.cuda.empty_cache()

    # ---------------------------------------------------------------- the attention forward, as bursts
    attention = None
    if not args.no_attention:
        attention = attention_entries(args, stream, peaks, dist, dev)

    # ---------------------------------------------------------------- end to end through the public API
    # Every step copies its inputs from pinned host memory, runs the GEMM and
    # copies C back; consecutive steps alternate between two CUDA streams, so
    # one step's copies overlap another step's GEMM.
    e2e_steps = max(3, min(K, args.e2e_steps))
    nstreams = 2
    tdt = head.tdt
    A_h = torch.from_numpy(head.A_bits.view(np.int16)).view(tdt).pin_memory()
    B_h = torch.from_numpy(head.B_bits.view(np.int16)).view(tdt).pin_memory()
    b_h = (torch.from_numpy(head.bias_bits.view(np.int16)).view(tdt).pin_memory()
           if head.bias_bits is not None else None)
    streams = [torch.cuda.Stream(dev) for _ in range(nstreams)]
    lanes = []
    for i in range(nstreams):
        Ad, Bd, Cd = head.sets[i % head.nsets]
        bd = torch.empty_like(head.bias) if head.bias is not None else None
        lanes.append((streams[i], Ad, Bd, bd, Cd, torch.empty((w.M, w.N), dtype=tdt).pin_memory()))

    def e2e_step(j):
        s, Ad, Bd, bd, Cd, C_h = lanes[j % nstreams]
        with torch.cuda.stream(s):
            Ad.copy_(A_h, non_blocking=True)
            Bd.copy_(B_h, non_blocking=True)
            if bd is not None:
                bd.copy_(b_h, non_blocking=True)
            tg.gemm(Ad, Bd, bd, epilogue=head.epi, out=Cd, stream=s)
            C_h.copy_(Cd, non_blocking=True)

    for j in range(2 * nstreams):
        e2e_step(j)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s_ in streams:
        s_.wait_event(e0)
    for j in range(e2e_steps):
        e2e_step(j)
    for s_ in streams:
        stream.wait_stream(s_)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    e2e_value = aggregate(w.flops * e2e_steps, e2e_ms / 1e3, ws) / 1e12
    h2d = 2 * (w.M * w.K + w.K * w.N) + (2 * w.N if head.bias_bits is not None else 0)
    d2h = 2 * w.M * w.N
    del lanes, A_h, B_h, b_h

    # ---------------------------------------------------------------- the headline, sustained
    sustained = None
    if args.sustained_s > 0:
        n = max(K, int(np.ceil(args.sustained_s / (kernel_ms / 1e3))))
        s_sampler = ClockSampler(local, period_s=0.01)
        s_ms = max_over_ranks(timed_region(head, stream, n, args.warmup, 0.0, sampler=s_sampler, dist=dist),
                              dist, dev)
        s_tflops = w.flops * n / (s_ms / 1e3) / 1e12
        s_peak, s_name = tensor_peak(peaks, s_ms / 1e3)
        sustained = {"steps": n, "region_s": round(s_ms / 1e3, 3), "tflops": round(s_tflops, 2),
                     "peak": s_peak, "frac": round(s_tflops / s_peak, 4), "peak_source": f"{peak_src} {s_name}",
                     "clocks": s_sampler.summary()}

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": ws, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(region_ms_max / K, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.DTYPE_NAMES[w.dtype], "data": "synthetic",
        "impl": "tl_gemm",
        "config": common_config(w, args.seed, ws),
        "kernel": {"config": head.plan["config_name"], "grid": head.plan["grid"], "split": head.plan["split"],
                   "raster_group": head.plan["raster_group"], "accumulate": "f32"},
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "streams": nstreams},
        "gpu_launches": K * head.launches_per_step,
        "clocks": clocks,
        "per_config": per_config,
        "attention": attention,
        "sustained": sustained,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, head.A_bits, head.B_bits, head.bias_bits, args.cpu_budget_s)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ the reference arm: the oracle
def run_reference(args, w):
    ws, rank, _ = dist_env()
    if rank != 0:
        return  # the oracle runs once, on rank 0's host cores
    import oracle
    A, B, bias = wl.make_inputs(w, args.seed)
    rows = oracle_sample_rows(w)
    # one step = one oracle call on the same row sample the cpu_baseline leg
    # times, so that the two CPU figures measure the same thing
    for _ in range(args.warmup):
        oracle_sample(w, A, B, bias, rows)
    t_tot = f_tot = 0.0
    for _ in range(args.steps):
        t, f = oracle_sample(w, A, B, bias, rows)
        t_tot += t
        f_tot += f
    value = f_tot / t_tot / 1e12
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t_tot / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": common_config(w, args.seed, ws),
        "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": oracle.max_threads(),
                         "sample": f"one oracle call per step on {len(rows)} of {w.M} rows of C "
                                   f"({len(rows)}x{w.N}x{w.K} multiply-adds, fp64)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=wl.HEADLINE, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="tl_gemm", choices=["tl_gemm", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ramp-s", type=float, default=0.01,
                    help="untimed back-to-back launches before the warm-up steps (brings the SM clock up)")
    ap.add_argument("--rest-s", type=float, default=1.5, help="idle time before each per-configuration burst")
    ap.add_argument("--sustained-s", type=float, default=3.0,
                    help="length of the sustained (power-capped) run of the headline; 0 skips it")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--no-attention", action="store_true")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be at least 3")
    if a.steps < 1:
        ap.error("--steps must be at least 1")
    return a


def main(argv=None):
    args = parse(argv)
    w = wl.WORKLOADS[args.workload]
    ws, _, _ = dist_env()
    if ws != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE={ws}; using WORLD_SIZE")
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)
    return 0


if __name__ == "__main__":
    sys.exit(main())
