"""bench.py on the GPU: a short run prints one JSON line with every key the
benchmark contract asks for, consistent with itself."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_short_bench_run_prints_the_contract_line():
    steps, warmup = 30, 3
    out = subprocess.run([sys.executable, "bench.py", "--steps", str(steps), "--warmup", str(warmup),
                          "--ramp-s", "0", "--no-cpu-baseline", "--e2e-steps", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == steps and d["warmup"] == warmup
    assert d["gpu_launches"] == steps and d["higher_is_better"] is True and d["data"] == "synthetic"
    assert d["config"]["workload"] == "gemm4096_f16"
    # the throughput follows from the step time: 2 M N K flops per step
    flops = 2 * 4096 ** 3
    assert abs(d["value"] - flops / (d["ms_per_step"] * 1e-3) / 1e12) <= 0.01 * d["value"]
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and 0 < r["frac"] < 1.2
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    # the committed ncu summary was taken on these kernel sources
    assert r["traffic"] is not None and r["traffic"] >= r["min_hbm_bytes_per_launch"]
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 2 * 2 * 4096 * 4096 and e["d2h_bytes_per_step"] == 2 * 4096 * 4096
    assert 0 < e["value"] <= d["value"]
    assert d["clocks"]["sm_max_mhz"] > 0
