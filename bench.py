#!/usr/bin/env python3
"""Benchmark of the fused tensor-core GEMM (libtlgemm.so) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one C = epilogue(A . B) call through the C ABI on the workload's
full size (default: 4096 x 4096 x 4096 fp16, no epilogue -- the GEMM the
TileLang pages benchmark).  Inputs are seeded synthetic data, resident in HBM
before the timed region; the timed region rotates over enough input/output
sets that every step reads operands that are not in L2.  Timing uses CUDA
events on the launching stream; with N > 1 (torchrun, one process per GPU)
each rank runs an independent replica (weak scaling, no data-path
collective) and the slowest rank's time counts.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle
instead (bounded row samples of the same workload on the host cores).
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
        except Exception as e:  # NVML missing: report no clocks rather than guess
            log("clock sampling unavailable:", e)
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
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
def oracle_rows_rate(w, A, B, bias, rows, repeats=1):
    """Seconds and flops for the oracle computing `rows` rows of C."""
    import oracle  # test infrastructure: the CPU-baseline leg only
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle.gemm(A, B, bias, w.dtype, w.epi, rows=rows)
    dt = time.perf_counter() - t0
    return dt, 2.0 * len(rows) * w.N * w.K * repeats


def cpu_baseline(w, A, B, bias, budget_s=12.0):
    """Oracle throughput on a bounded sample of rows, sized for ~budget_s."""
    import oracle
    rng = np.random.default_rng(0)
    # each call has a fixed cost (decoding B) plus a cost per row: time two
    # sizes and size the sample from the marginal cost per row
    small = np.sort(rng.choice(w.M, size=min(4, w.M), replace=False))
    large = np.sort(rng.choice(w.M, size=min(32, w.M), replace=False))
    t1, _ = oracle_rows_rate(w, A, B, bias, small)
    t2, _ = oracle_rows_rate(w, A, B, bias, large)
    per_row = max((t2 - t1) / max(len(large) - len(small), 1), t2 / len(large) / 8, 1e-9)
    fixed = max(t1 - per_row * len(small), 0.0)
    n = int(max(1, min(w.M, (budget_s - fixed) / per_row)))
    rows = np.sort(rng.choice(w.M, size=n, replace=False))
    t, f = oracle_rows_rate(w, A, B, bias, rows)
    return {"value": f / t / 1e12, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{n} of {w.M} rows of C ({n}x{w.N}x{w.K} multiply-adds, fp64), {t:.1f} s"}


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


def run_gpu(args, w):
    import torch
    ws, rank, local = dist_env()
    dist = init_dist("nccl", ws)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    ensure_library()
    import tensor_core_gemm_tl_b200 as tg

    A_bits, B_bits, bias_bits = wl.make_inputs(w, args.seed)
    tdt = torch.float16 if w.dtype == wl.F16 else torch.bfloat16

    def dev_tensor(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(tdt)

    A0, B0 = dev_tensor(A_bits), dev_tensor(B_bits)
    bias0 = dev_tensor(bias_bits) if bias_bits is not None else None
    set_bytes = 2 * (w.M * w.K + w.K * w.N + w.M * w.N)
    nsets = max(2, int(np.ceil(3 * L2_BYTES / set_bytes)))
    sets = []
    for i in range(nsets):
        A = A0 if i == 0 else A0.clone()
        B = B0 if i == 0 else B0.clone()
        C = torch.empty((w.M, w.N), dtype=tdt, device=dev)
        sets.append((A, B, C))
    stream = torch.cuda.current_stream(dev)
    epi = "bias_gelu" if w.epi == wl.EPI_BIAS_GELU else None

    plan = tg.plan(w.M, w.N, w.K, w.dtype, epi, num_sms=torch.cuda.get_device_properties(dev).multi_processor_count,
                   ptrs=(sets[0][0].data_ptr(), sets[0][1].data_ptr(),
                         bias0.data_ptr() if bias0 is not None else 0, sets[0][2].data_ptr()))
    launches_per_step = 1 + plan["pad_a"] + plan["pad_b"]

    def step(i):
        A, B, C = sets[i % nsets]
        tg.gemm(A, B, bias0, epilogue=epi, out=C, stream=stream)

    # bring clocks up, then the W untimed warm-up steps
    t_end = time.time() + args.ramp_s
    i = 0
    while time.time() < t_end:
        for _ in range(20):
            step(i)
            i += 1
        torch.cuda.synchronize()
    for j in range(args.warmup):
        step(j)
    torch.cuda.synchronize()
    if tg.check_device() != 0:
        raise RuntimeError("device error during warm-up")

    K = args.steps
    # Events only at the two ends of the region: an event between launches
    # would serialise them and hide the overlap of one kernel's set-up with the
    # previous kernel's tail.  The kernel's average launch duration is then the
    # region time over the launches in it (gaps included, so it errs low).
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        t_start.record(stream)
        for j in range(K):
            step(j)
        t_end.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    region_ms = t_start.elapsed_time(t_end)
    if tg.check_device() != 0:
        raise RuntimeError("device error in the timed region")
    region_ms_max = max_over_ranks(region_ms, dist, dev)
    gemm_launches = K  # the GEMM kernel runs once per step
    kernel_ms = region_ms / gemm_launches

    value = aggregate(w.flops * K, region_ms_max / 1e3, ws) / 1e12

    # End to end through the public API, the way a caller streams work through
    # it: every step copies its inputs from pinned host memory, runs the GEMM and
    # copies C back; consecutive steps alternate between two CUDA streams, so
    # one step's copies overlap another step's GEMM.
    e2e_steps = max(3, min(K, args.e2e_steps))
    nstreams = 2
    A_h = torch.from_numpy(A_bits.view(np.int16)).view(tdt).pin_memory()
    B_h = torch.from_numpy(B_bits.view(np.int16)).view(tdt).pin_memory()
    b_h = torch.from_numpy(bias_bits.view(np.int16)).view(tdt).pin_memory() if bias_bits is not None else None
    streams = [torch.cuda.Stream(dev) for _ in range(nstreams)]
    lanes = []
    for i in range(nstreams):
        Ad, Bd, Cd = sets[i % nsets]
        bd = torch.empty_like(bias0) if bias0 is not None else None
        lanes.append((streams[i], Ad, Bd, bd, Cd, torch.empty((w.M, w.N), dtype=tdt).pin_memory()))

    def e2e_step(j):
        s, Ad, Bd, bd, Cd, C_h = lanes[j % nstreams]
        with torch.cuda.stream(s):
            Ad.copy_(A_h, non_blocking=True)
            Bd.copy_(B_h, non_blocking=True)
            if bd is not None:
                bd.copy_(b_h, non_blocking=True)
            tg.gemm(Ad, Bd, bd, epilogue=epi, out=Cd, stream=s)
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
    h2d = 2 * (w.M * w.K + w.K * w.N) + (2 * w.N if bias_bits is not None else 0)
    d2h = 2 * w.M * w.N

    peaks, peak_src = measured_peaks()
    # fp16 and bf16 share the dense tensor rate.  A timed region that runs under
    # sustained load (the clock ramp plus the region last a second or more) is
    # compared with the sustained figure, a short burst with the burst figure.
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    long_run = args.ramp_s + region_ms_max / 1e3 >= 1.0
    peak = sustained if long_run else burst
    peak_name = "bf16_tflops_sustained (back-to-back cuBLAS loop)" if long_run else "bf16_tflops (burst, cuBLAS)"
    achieved = w.flops / (kernel_ms / 1e3) / 1e12
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": ws, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(region_ms_max / K, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.DTYPE_NAMES[w.dtype], "data": "synthetic",
        "impl": "tl_gemm",
        "config": {**w.describe(), "kernel_config": plan["config_name"], "grid": plan["grid"],
                   "parallelism": f"replicas{ws}" if ws > 1 else "single",
                   "l2": f"rotating {nsets} input/output sets of {set_bytes / 2**20:.0f} MiB "
                         f"({nsets * set_bytes / 2**20:.0f} MiB > {L2_BYTES / 2**20:.0f} MiB L2)",
                   "accumulate": "f32", "seed": args.seed},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": UNIT,
                     "frac": round(achieved / peak, 4), "traffic": ncu_traffic(w.name),
                     "peak_source": f"{peak_src} {peak_name}; fp16 dense rate equals bf16",
                     "frac_of_burst_peak": round(achieved / burst, 4),
                     "kernel_ms": round(kernel_ms, 5), "kernel_ms_is": "timed region / launches",
                     "algorithmic_flops_per_launch": w.flops,
                     "min_hbm_bytes_per_launch": w.min_bytes()},
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "streams": nstreams},
        "gpu_launches": K * launches_per_step,
        "clocks": sampler.summary(),
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, A_bits, B_bits, bias_bits, args.cpu_budget_s)
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
    rng = np.random.default_rng(1)

    def points(n):
        return rng.integers(0, w.M, n), rng.integers(0, w.N, n)

    def timed(n):
        ii, jj = points(n)
        t0 = time.perf_counter()
        oracle.gemm_points(A, B, bias, w.dtype, w.epi, ii, jj)
        return time.perf_counter() - t0

    # one step = `n` single elements of C (2K flops each) through the oracle's
    # element entry point, sized so that all steps fit in about ref_budget_s
    timed(256)
    per_point = max(timed(2048) / 2048, 1e-9)
    total_steps = args.steps + args.warmup
    n = int(max(64, min(w.M * w.N, args.ref_budget_s / total_steps / per_point)))
    for _ in range(args.warmup):
        timed(n)
    t_tot = 0.0
    for _ in range(args.steps):
        t_tot += timed(n)
    f_tot = 2.0 * w.K * n * args.steps
    value = f_tot / t_tot / 1e12
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t_tot / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {**w.describe(), "seed": args.seed},
        "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": oracle.max_threads(),
                         "sample": f"{n} random elements of C per step (2K flops each), fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=wl.HEADLINE, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="tl_gemm", choices=["tl_gemm", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ramp-s", type=float, default=1.0, help="untimed clock ramp before the warm-up steps")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--ref-budget-s", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
