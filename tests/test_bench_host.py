"""Host-side logic of bench.py on the CPU: the multi-rank aggregation (max of
the per-rank times, whole-job throughput) with two gloo ranks, the argument
contract, and the JSON of the reference arm."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    d = bench.init_dist("gloo", world)
    # rank r "took" (r + 1) * 10 ms for the same units of work
    t = bench.max_over_ranks(0.010 * (rank + 1), d)
    value = bench.aggregate(units_per_rank=1000.0, seconds_max=t, world=world)
    dist.barrier()
    dist.destroy_process_group()
    out_q.put((rank, t, value))


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, value in res:
        assert t == pytest.approx(0.020)              # the max over ranks
        assert value == pytest.approx(2 * 1000 / 0.020)  # all ranks' units / max time


def test_single_process_needs_no_process_group():
    assert bench.max_over_ranks(1.5, None) == 1.5
    assert bench.aggregate(10.0, 2.0, 1) == 5.0


def test_argument_contract():
    a = bench.parse([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1
    assert a.workload == "mlp_up_8192x16384x4096_bf16_bias_gelu"  # the largest configuration
    with pytest.raises(SystemExit):
        bench.parse(["--warmup", "2"])


def test_reference_arm_json_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "gemm256_f16_bias_gelu", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "gemm256_f16_bias_gelu"
    # the same workload keys the GPU arm prints
    assert d["config"] == bench.common_config(bench.wl.WORKLOADS["gemm256_f16_bias_gelu"], 0, 1)


def test_reference_arm_other_ranks_print_nothing():
    env = dict(os.environ, PYTHONPATH=ROOT, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "gemm256_f16_bias_gelu", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_traffic_is_tied_to_the_kernel_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = bench.kernel_source_hash()
    (prof / "x.md").write_text(f"<!-- traffic workload=w1 src={src} bytes_per_launch=123 -->\n"
                               f"<!-- traffic workload=w2 src=deadbeef bytes_per_launch=456 -->\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: src)
    assert bench.ncu_traffic("w1") == 123
    assert bench.ncu_traffic("w2") is None


def test_attention_flop_count_closed_forms():
    """The attention figures count 4 D flops per kept (query, key) pair: all
    Sq Sk pairs without a mask; with the causal mask (key j <= query i) row i
    keeps min(i + 1, Sk) keys, whose sum has a closed form for Sq <= Sk (a
    triangle) and for Sq > Sk (a triangle plus full rows)."""
    from tensor_core_gemm_tl_b200.compare import attention_flops
    B, H, D = 3, 5, 64
    assert attention_flops(B, H, 4096, 4096, D, False) == 4 * B * H * D * 4096 * 4096
    assert attention_flops(B, H, 4096, 4096, D, True) == 4 * B * H * D * 4096 * 4097 // 2
    Sq, Sk = 300, 1000  # every row sees i + 1 keys
    assert attention_flops(B, H, Sq, Sk, D, True) == 4 * B * H * D * Sq * (Sq + 1) // 2
    Sq, Sk = 1000, 300  # rows past Sk - 1 see all Sk keys
    kept = Sk * (Sk + 1) // 2 + (Sq - Sk) * Sk
    assert attention_flops(B, H, Sq, Sk, D, True) == 4 * B * H * D * kept


def test_peak_follows_the_timed_region_length():
    """A region shorter than a second is a burst (burst peak); a longer one
    runs power-capped (sustained peak)."""
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    assert bench.tensor_peak(peaks, 0.015) == (1600.0, "bf16_tflops")
    assert bench.tensor_peak(peaks, 0.999) == (1600.0, "bf16_tflops")
    assert bench.tensor_peak(peaks, 1.0) == (1400.0, "bf16_tflops_sustained")
    assert bench.tensor_peak({"bf16_tflops": 1600.0, "hbm_gbs": 6500.0}, 5.0)[0] == 1600.0


def test_bound_of_each_benchmark_configuration():
    """Roofline class per configuration: launch latency for 256^3, HBM for
    the 128-row skinny shape, the tensor pipe for the rest."""
    wl = bench.wl
    got = {n: bench.bound_of(wl.WORKLOADS[n]) for n in bench.PER_CONFIG}
    for n, b in got.items():
        w = wl.WORKLOADS[n]
        expect = "latency" if w.M == 256 else ("hbm" if w.M == 128 else "tensor")
        assert b == expect, (n, b)


def test_oracle_sample_is_the_same_for_both_cpu_figures():
    """cpu_baseline and the reference arm time the same row sample: a fixed
    number of multiply-adds, rows drawn without replacement."""
    wl = bench.wl
    for n in bench.PER_CONFIG:
        w = wl.WORKLOADS[n]
        r1, r2 = bench.oracle_sample_rows(w), bench.oracle_sample_rows(w)
        assert (r1 == r2).all() and len(set(r1.tolist())) == len(r1) and r1.max() < w.M
        assert len(r1) == max(1, min(w.M, round(bench.ORACLE_SAMPLE_MACS / (w.N * w.K))))
