"""Time the library against PyTorch eager on the same workloads (needs a GPU).

The TileLang pages compare their GEMM with PyTorch and cuBLAS, and their
fused bias + GELU epilogue with PyTorch eager (TileLang GPU kernel design
article, paragraphs 2 and 5).  This tool does the same on a B200: for each
named workload it times

  * tl_gemm (this library, through the C ABI),
  * torch.matmul (cuBLAS), and for the epilogue workloads
  * torch eager  A @ B + bias, then torch.nn.functional.gelu (exact form):
    three kernels and two intermediates through HBM,

with CUDA events over operands rotated beyond L2, median of the launches.
It prints one JSON line per workload.  A diagnostic, not the benchmark.

    python -m tensor_core_gemm_tl_b200.compare [--only name,...] [--launches 40] [--attention]

With --attention it times tl_attention_fwd against PyTorch's
scaled_dot_product_attention (bf16, random inputs) on a few
transformer-sized shapes; with --rowwise, the row softmax and the vector add
as achieved HBM GB/s against torch.softmax and torch.add.
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

L2_BYTES = 126 * 1024 * 1024


def _median_ms(fn, nsets, launches, warmup):
    import torch
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        fn(i % nsets)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
    for i, (s, e) in enumerate(ev):
        s.record(stream)
        fn(i % nsets)
        e.record(stream)
    torch.cuda.synchronize()
    return float(np.median([s.elapsed_time(e) for s, e in ev]))


def compare(w, launches=40, warmup=10):
    import torch
    import torch.nn.functional as F
    import tensor_core_gemm_tl_b200 as tg
    A_bits, B_bits, bias_bits = wl.make_inputs(w, 0)
    tdt = torch.float16 if w.dtype == wl.F16 else torch.bfloat16

    def dev(bits):
        return torch.from_numpy(bits.view(np.int16)).cuda().view(tdt)

    A0, B0 = dev(A_bits), dev(B_bits)
    bias = dev(bias_bits) if bias_bits is not None else None
    set_bytes = 2 * (w.M * w.K + w.K * w.N + w.M * w.N)
    nsets = max(2, int(np.ceil(3 * L2_BYTES / set_bytes)))
    sets = [(A0.clone(), B0.clone(), torch.empty((w.M, w.N), dtype=tdt, device="cuda")) for _ in range(nsets)]
    epi = "bias_gelu" if w.epi == wl.EPI_BIAS_GELU else None

    def ours(i):
        A, B, C = sets[i]
        tg.gemm(A, B, bias, epilogue=epi, out=C)

    def cublas(i):
        A, B, C = sets[i]
        torch.matmul(A, B, out=C)

    def eager(i):
        A, B, C = sets[i]
        C.copy_(F.gelu(torch.matmul(A, B) + bias, approximate="none"))

    res = {"workload": w.name, "M": w.M, "N": w.N, "K": w.K}
    t = _median_ms(ours, nsets, launches, warmup)
    res["tl_gemm_tflops"] = round(w.flops / t / 1e9, 1)
    t = _median_ms(cublas, nsets, launches, warmup)
    res["torch_matmul_tflops"] = round(w.flops / t / 1e9, 1)
    if epi:
        t = _median_ms(eager, nsets, launches, warmup)
        res["torch_eager_bias_gelu_tflops"] = round(w.flops / t / 1e9, 1)
    if tg.check_device() != 0:
        raise RuntimeError("device error")
    return res


def attention_flops(B, H, Sq, Sk, D, causal):
    """4 D flops per kept (query, key) pair: Q K^T and P V."""
    if causal:
        kept = sum(min(i + 1, Sk) for i in range(Sq))
    else:
        kept = Sq * Sk
    return 4.0 * B * H * D * kept


ATTENTION_SHAPES = [
    # B, H, Sq, Sk, D, causal
    (4, 16, 4096, 4096, 128, False),
    (4, 16, 4096, 4096, 128, True),
    (8, 16, 2048, 2048, 64, False),
    (8, 16, 2048, 2048, 64, True),
    (1, 32, 8192, 8192, 128, True),
]


def compare_attention(B, H, Sq, Sk, D, causal, launches=20, warmup=5):
    import torch
    import torch.nn.functional as F
    import tensor_core_gemm_tl_b200 as tg
    g = torch.Generator(device="cuda").manual_seed(0)
    q = torch.randn(B, H, Sq, D, device="cuda", dtype=torch.bfloat16, generator=g)
    k = torch.randn(B, H, Sk, D, device="cuda", dtype=torch.bfloat16, generator=g)
    v = torch.randn(B, H, Sk, D, device="cuda", dtype=torch.bfloat16, generator=g)
    out = torch.empty_like(q)

    def ours(_):
        tg.attention(q, k, v, causal=causal, out=out)

    def sdpa(_):
        F.scaled_dot_product_attention(q, k, v, is_causal=causal)

    fl = attention_flops(B, H, Sq, Sk, D, causal)
    res = {"attention": f"B{B} H{H} Sq{Sq} Sk{Sk} D{D}", "causal": causal, "dtype": "bf16"}
    res["tl_attention_tflops"] = round(fl / _median_ms(ours, 1, launches, warmup) / 1e9, 1)
    res["torch_sdpa_tflops"] = round(fl / _median_ms(sdpa, 1, launches, warmup) / 1e9, 1)
    if tg.check_device() != 0:
        raise RuntimeError("device error")
    return res


ROWWISE_SHAPES = [(16384, 8192), (65536, 1024), (4096, 50257), (262144, 128)]


def compare_rowwise(launches=20, warmup=5, shapes=ROWWISE_SHAPES, vector_n=1 << 28):
    """Achieved HBM bandwidth (compulsory bytes / time) of the row softmax and
    the vector add against torch.softmax and torch.add (vector_n = 0 skips
    the vector add)."""
    import torch
    import tensor_core_gemm_tl_b200 as tg
    out = []
    for rows, cols in shapes:
        x = torch.randn(rows, cols, device="cuda", dtype=torch.bfloat16)
        y = torch.empty_like(x)
        nbytes = 2 * 2 * rows * cols

        def ours(_):
            tg.softmax(x, out=y)

        def ref(_):
            torch.softmax(x, dim=-1, out=y)

        out.append({"softmax": f"{rows}x{cols} bf16",
                    "tl_gbs": round(nbytes / _median_ms(ours, 1, launches, warmup) / 1e6, 1),
                    "torch_gbs": round(nbytes / _median_ms(ref, 1, launches, warmup) / 1e6, 1)})
    n = vector_n
    if n <= 0:
        if tg.check_device() != 0:
            raise RuntimeError("device error")
        return out
    a = torch.randn(n, device="cuda")
    b = torch.randn(n, device="cuda")
    c = torch.empty_like(a)

    def ours_add(_):
        tg.vector_add(a, b, out=c)

    def ref_add(_):
        torch.add(a, b, out=c)

    nbytes = 3 * 4 * n
    out.append({"vector_add": f"{n} float32",
                "tl_gbs": round(nbytes / _median_ms(ours_add, 1, launches, warmup) / 1e6, 1),
                "torch_gbs": round(nbytes / _median_ms(ref_add, 1, launches, warmup) / 1e6, 1)})
    if tg.check_device() != 0:
        raise RuntimeError("device error")
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", default=None)
    ap.add_argument("--launches", type=int, default=40)
    ap.add_argument("--attention", action="store_true", help="time attention forward instead of the GEMMs")
    ap.add_argument("--rowwise", action="store_true", help="time the row softmax and the vector add")
    ap.add_argument("--rowwise-shapes", default=None,
                    help="comma-separated ROWSxCOLS softmax shapes (default: the four standard ones)")
    ap.add_argument("--vector-n", type=int, default=1 << 28, help="vector add length (0: skip it)")
    a = ap.parse_args(argv)
    import torch
    torch.cuda.set_device(0)
    if a.attention:
        for shape in ATTENTION_SHAPES:
            print(json.dumps(compare_attention(*shape)), flush=True)
        return 0
    if a.rowwise:
        shapes = ROWWISE_SHAPES
        if a.rowwise_shapes is not None:
            shapes = [tuple(int(v) for v in x.split("x")) for x in a.rowwise_shapes.split(",") if x]
        for rec in compare_rowwise(launches=min(a.launches, 20), shapes=shapes, vector_n=a.vector_n):
            print(json.dumps(rec), flush=True)
        return 0
    todo = list(wl.WORKLOADS.values())
    if a.only:
        keep = set(a.only.split(","))
        todo = [w for w in todo if w.name in keep]
    for w in todo:
        print(json.dumps(compare(w, a.launches)), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
