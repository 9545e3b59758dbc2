"""Offline tile/stage configuration sweep (needs a B200).

For each shape, every compiled kernel configuration (with and without the
split last round, and with each raster group asked for) is timed through
tl_gemm_ex on seeded inputs: rotating over input sets larger than L2, a short
region of back-to-back launches between two CUDA events after an idle pause,
so that it runs at the unthrottled clock, as the benchmark's bursts do.  With --write, the fastest
configuration per (M, N, K, dtype, epilogue) is written to
csrc/config_table.inc, which the library compiles in; shapes not in the table
use the library's wave model.  Nothing here runs at call time.

    python -m tensor_core_gemm_tl_b200.sweep [--write] [--launches 20] [--shapes all|named] [--groups 0,4,16]
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

TABLE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc", "config_table.inc")
L2_BYTES = 126 * 1024 * 1024


class Operands:
    """Rotating input/output sets of one workload (together larger than L2)."""

    def __init__(self, w, seed=0):
        import torch
        A_bits, B_bits, bias_bits = wl.make_inputs(w, seed)
        tdt = torch.float16 if w.dtype == wl.F16 else torch.bfloat16

        def dev(bits):
            return torch.from_numpy(bits.view(np.int16)).cuda().view(tdt)

        A0, B0 = dev(A_bits), dev(B_bits)
        self.bias = dev(bias_bits) if bias_bits is not None else None
        set_bytes = 2 * (w.M * w.K + w.K * w.N + w.M * w.N)
        self.nsets = max(2, int(np.ceil(3 * L2_BYTES / set_bytes)))
        self.sets = [(A0 if i == 0 else A0.clone(), B0 if i == 0 else B0.clone(),
                      torch.empty((w.M, w.N), dtype=tdt, device="cuda")) for i in range(self.nsets)]
        self.epi = "bias_gelu" if w.epi == wl.EPI_BIAS_GELU else None


def time_config(ops, config, launches, warmup, no_split=False, raster_group=0, rest_s=0.5, force_split=False):
    """Average milliseconds per launch of `launches` back-to-back launches
    (two events around the whole region), after `rest_s` of idle time and
    `warmup` launches, so that the region runs at the unthrottled clock."""
    import time
    import torch
    import tensor_core_gemm_tl_b200 as tg
    stream = torch.cuda.current_stream()

    def launch(i):
        A, B, C = ops.sets[i % ops.nsets]
        tg.gemm(A, B, ops.bias, epilogue=ops.epi, out=C, config=config, stream=stream, no_split=no_split,
                raster_group=raster_group, force_split=force_split)

    torch.cuda.synchronize()
    time.sleep(rest_s)
    for i in range(warmup):
        launch(i)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(launches):
        launch(i)
    t1.record(stream)
    torch.cuda.synchronize()
    if tg.check_device() != 0:
        raise RuntimeError("device error")
    return t0.elapsed_time(t1) / launches


def shapes(which):
    named = list(wl.WORKLOADS.values())
    if which == "named":
        return named
    extra = [wl.custom(f"square{n}_{d}", n, n, n, dt, 0) for n in (1024, 2048, 8192)
             for d, dt in (("f16", wl.F16), ("bf16", wl.BF16))]
    return named + extra


def read_table(path=TABLE):
    """The rows of an existing table as records (shape, config, split, group, TFLOP/s)."""
    import re
    rows = []
    if not os.path.exists(path):
        return rows
    pat = re.compile(r'\{(\d+), (\d+), (\d+), (\d+), (\d+), "([^"]+)", (\d+)(?:, (\d+))?\},\s*//\s*([\d.]+) TFLOP/s')
    for m in pat.finditer(open(path).read()):
        M, N, K, dt, epi = (int(m.group(i)) for i in range(1, 6))
        rows.append({"M": M, "N": N, "K": K, "dtype": "f16" if dt == 0 else "bf16", "epi": epi,
                     "config": m.group(6), "split": int(m.group(7)), "group": int(m.group(8) or 0),
                     "tflops": float(m.group(9))})
    return rows


def merge_rows(new_rows, old_rows):
    """The new rows, then the old rows for shapes the new sweep did not time."""
    key = lambda r: (r["M"], r["N"], r["K"], r["dtype"], r["epi"])  # noqa: E731
    seen = {key(r) for r in new_rows}
    return list(new_rows) + [r for r in old_rows if key(r) not in seen]


def write_table(best_rows):
    """Write csrc/config_table.inc from the fastest record per shape."""
    lines = ["// Kernel configuration per measured shape: {M, N, K, dtype, epilogue, config, split, raster group}.",
             "// Written by tensor_core_gemm_tl_b200/sweep.py from timings on a B200; shapes",
             "// not listed fall back to the wave model in tl_gemm.cu."]
    seen = set()
    for r in best_rows:
        key = (r["M"], r["N"], r["K"], r["dtype"], r["epi"])
        if key in seen:
            continue
        seen.add(key)
        dt = 0 if r["dtype"] == "f16" else 1
        split = int(r.get("split", 0))
        group = int(r.get("group", 0))
        lines.append(f'{{{r["M"]}, {r["N"]}, {r["K"]}, {dt}, {r["epi"]}, "{r["config"]}", {split}, {group}}},'
                     f'  // {r["tflops"]} TFLOP/s')
    lines.append('{0, 0, 0, -1, -1, "", 0, 0},  // sentinel, never matches')
    with open(TABLE, "w") as f:
        f.write("\n".join(lines) + "\n")
    print("wrote", TABLE, file=sys.stderr)


def best_from_records(records):
    """The fastest record (lowest median time) per workload, in input order."""
    best = {}
    for r in records:
        k = r["workload"]
        if k not in best or r["median_ms"] < best[k]["median_ms"]:
            best[k] = r
    return list(best.values())


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--write", action="store_true")
    ap.add_argument("--launches", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--rest-s", type=float, default=0.5, help="idle time before each timed region")
    ap.add_argument("--groups", default="0", help="comma-separated raster groups to try (0: the library's choice)")
    ap.add_argument("--configs", default=None, help="comma-separated 1-based configurations to try (default: all)")
    ap.add_argument("--shapes", default="named", choices=["named", "all"])
    ap.add_argument("--only", default=None, help="comma-separated workload names")
    ap.add_argument("--from-jsonl", default=None, help="write the table from recorded sweep output")
    a = ap.parse_args(argv)
    a.groups = [int(x) for x in a.groups.split(",")]
    if a.from_jsonl:
        with open(a.from_jsonl) as f:
            write_table(merge_rows(best_from_records([json.loads(x) for x in f if x.strip()]), read_table()))
        return 0
    import torch
    import tensor_core_gemm_tl_b200 as tg
    torch.cuda.set_device(0)
    rows = []
    todo = shapes(a.shapes)
    if a.only:
        keep = set(a.only.split(","))
        todo = [w for w in todo if w.name in keep]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for w in todo:
        ops = Operands(w)
        best = None
        for k in ([int(x) for x in a.configs.split(",")] if a.configs else range(1, tg.tl_num_configs() + 1)):
            p = tg.plan(w.M, w.N, w.K, w.dtype, ops.epi, num_sms=sms, config=k, force_split=True)
            for split in ((1, 0) if p["split"] > 1 else (0,)):
                for group in a.groups:
                    ms = time_config(ops, k, a.launches, a.warmup, no_split=not split, raster_group=group,
                                     rest_s=a.rest_s, force_split=bool(split))
                    tflops = w.flops / (ms / 1e3) / 1e12
                    rec = {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "dtype": wl.DTYPE_NAMES[w.dtype],
                           "epi": w.epi, "config": tg.tl_config_name(k - 1), "config_index": k - 1, "split": split,
                           "group": group, "median_ms": round(ms, 5), "tflops": round(tflops, 1)}
                    print(json.dumps(rec), flush=True)
                    if best is None or ms < best[0]:
                        best = (ms, rec)
        rows.append(best[1])
        del ops
        torch.cuda.empty_cache()
    if a.write:
        write_table(merge_rows(rows, read_table()))
    return 0


if __name__ == "__main__":
    sys.exit(main())
