"""bench.py on the GPU: a short run prints one JSON line with every key the
benchmark contract asks for, consistent with itself."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_short_bench_run_prints_the_contract_line():
    import bench
    import workloads as wl
    steps, warmup = 20, 3
    out = subprocess.run([sys.executable, "bench.py", "--steps", str(steps), "--warmup", str(warmup),
                          "--no-cpu-baseline", "--e2e-steps", "3", "--rest-s", "0.05", "--sustained-s", "0.3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
                "per_config", "attention", "sustained"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == steps and d["warmup"] == warmup
    assert d["gpu_launches"] == steps and d["higher_is_better"] is True and d["data"] == "synthetic"
    w = wl.WORKLOADS["mlp_up_8192x16384x4096_bf16_bias_gelu"]
    assert d["config"]["workload"] == w.name and d["dtype"] == "bf16"
    assert d["config"] == bench.common_config(w, 0, 1)
    # the throughput follows from the step time: 2 M N K flops per step
    assert abs(d["value"] - w.flops / (d["ms_per_step"] * 1e-3) / 1e12) <= 0.01 * d["value"]
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and 0 < r["frac"] < 1.2
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    # a region of milliseconds is a burst: compared with the burst peak
    peaks, _ = bench.measured_peaks()
    assert r["region_s"] < 1.0 and r["peak"] == float(peaks["bf16_tflops"])
    # a traffic figure, when the committed ncu summary matches these sources, is at least the compulsory bytes
    assert r["traffic"] is None or r["traffic"] >= 0.9 * r["min_hbm_bytes_per_launch"]
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 2 * (w.M * w.K + w.K * w.N) + 2 * w.N
    assert e["d2h_bytes_per_step"] == 2 * w.M * w.N
    assert 0 < e["value"] <= d["value"]
    assert d["clocks"]["sm_max_mhz"] > 0 and d["clocks"]["samples"] >= 1
    # every configuration of the benchmark set, each self-consistent
    assert set(d["per_config"]) == set(bench.PER_CONFIG)
    for name, c in d["per_config"].items():
        wc = wl.WORKLOADS[name]
        assert abs(c["tflops"] - wc.flops / (c["ms"] * 1e-3) / 1e12) <= 0.01 * c["tflops"] + 0.01, name
        assert abs(c["gbs"] - wc.min_bytes() / (c["ms"] * 1e-3) / 1e9) <= 0.01 * c["gbs"] + 0.1, name
        expect = "hbm" if name.startswith("skinny") else ("latency" if wc.M == 256 else "tensor")
        assert c["bound"] == expect, name
        assert c["warm_l2_tflops"] > 0
    s = d["sustained"]
    assert s["steps"] >= steps and s["tflops"] > 0
    # the attention forward beside the GEMMs, each entry self-consistent
    assert len(d["attention"]) == len(bench.ATTENTION_SHAPES)
    for name, a in d["attention"].items():
        assert a["tflops"] > 0 and a["torch_sdpa_tflops"] > 0, name
        assert abs(a["frac"] - a["tflops"] / float(peaks["bf16_tflops"])) < 1e-3, name
