"""tl_gemm_noalloc: the entry point for callers that cannot allocate device
memory (an inference engine's plugin whose execute step must not allocate, a
service holding a fixed memory budget, code that must not synchronize the
device or break a stream capture with cudaMalloc).  It must give what tl_gemm
gives, call after call, keep its padded copies in the library's fixed scratch
area, refuse work that needs more than that area, and allocate nothing.

This file is collected last on purpose, and it is self-contained: it passes
alone in a fresh process as well as after the rest of the suite.
"""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import workloads as wl  # noqa: E402
from gpu_util import compare, from_device, to_device, torch_dtype  # noqa: E402

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

SCRATCH_BYTES = 64 << 20


def _buffers(A_bits, B_bits, bias_bits, dt):
    A, B = to_device(A_bits, dt), to_device(B_bits, dt)
    bias = to_device(bias_bits, dt) if bias_bits is not None else None
    out = torch.empty((A_bits.shape[0], B_bits.shape[1]), dtype=torch_dtype(dt), device="cuda")
    return A, B, bias, out


def _run(entry, bufs, dt, epi):
    import tensor_core_gemm_tl_b200 as tg
    A, B, bias, out = bufs
    M, K = A.shape
    N = B.shape[1]
    stream = torch.cuda.current_stream().cuda_stream
    st = entry(A.data_ptr(), B.data_ptr(), bias.data_ptr() if bias is not None else 0, out.data_ptr(),
               M, N, K, dt, epi, stream)
    assert st == 0, tg.tl_status_string(st)
    assert tg.check_device() == 0
    return from_device(out)


# (M, N, K, dtype, epilogue, what the plan puts in the scratch area)
CASES = [
    # A and B copied into zero-padded scratch, C stored element by element, and
    # the last round split: partial sums and arrival words in scratch too
    (300, 1001, 2050, wl.BF16, wl.EPI_BIAS_GELU, "pad_a pad_b split"),
    # only A padded (K = 300); too few k-blocks to split
    (2048, 2048, 300, wl.F16, wl.EPI_BIAS_GELU, "pad_a"),
    # aligned operands and whole rounds of tiles: no scratch at all
    (2048, 2048, 2048, wl.BF16, wl.EPI_NONE, ""),
    # aligned operands, split last round: scratch for the partial sums only
    (1024, 1024, 2048, wl.BF16, wl.EPI_BIAS_GELU, "split"),
]


def _plan(M, N, K, dt, epi, bufs):
    import tensor_core_gemm_tl_b200 as tg
    A, B, bias, out = bufs
    st, p = tg.tl_gemm_plan(A.data_ptr(), B.data_ptr(), bias.data_ptr() if bias is not None else 0,
                            out.data_ptr(), M, N, K, dt, epi, 0)
    assert st == 0
    return p


def _check_plan_kind(p, kind):
    uses = set(kind.split())
    assert bool(p.pad_a) == ("pad_a" in uses) and bool(p.pad_b) == ("pad_b" in uses)
    assert (p.split > 1) == ("split" in uses)
    assert (p.workspace_bytes > 0) == bool(uses)
    assert p.workspace_bytes <= SCRATCH_BYTES


@pytest.mark.parametrize("M,N,K,dt,epi,kind", CASES)
def test_noalloc_matches_tl_gemm_on_two_calls_in_a_row(M, N, K, dt, epi, kind):
    import tensor_core_gemm_tl_b200 as tg
    for seed in (11, 12):  # two calls in a row, the second on new inputs
        A, B, bias = wl.make_inputs(wl.custom("noalloc", M, N, K, dt, epi), seed)
        bufs = _buffers(A, B, bias, dt)
        _check_plan_kind(_plan(M, N, K, dt, epi, bufs), kind)
        expected = _run(tg.tl_gemm, bufs, dt, epi)
        got = _run(tg.tl_gemm_noalloc, bufs, dt, epi)
        # within the suite's tolerances of the existing entry point's result ...
        compare(got, wl.bits_to_float32(expected, dt).astype(np.float64), dt)
        # ... and in fact identical: the same kernels and configuration run
        assert np.array_equal(got, expected)


def test_noalloc_refuses_work_beyond_its_scratch_and_enqueues_nothing():
    import tensor_core_gemm_tl_b200 as tg
    M, N, K = 20000, 64, 2050  # A padded to 20000 x 2112 x 2 bytes > 64 MiB
    st, plan = tg.tl_gemm_plan(256, 256, 0, 256, M, N, K, wl.BF16, wl.EPI_NONE, 148)
    assert st == 0 and plan.workspace_bytes > SCRATCH_BYTES
    A, B, _ = wl.make_inputs(wl.custom("big", M, N, K, wl.BF16, wl.EPI_NONE), 1)
    bufs = list(_buffers(A, B, None, wl.BF16))
    bufs[3].fill_(3.0)
    Ad, Bd, _, out = bufs
    torch.cuda.synchronize()
    st = tg.tl_gemm_noalloc(Ad.data_ptr(), Bd.data_ptr(), 0, out.data_ptr(), M, N, K, wl.BF16, wl.EPI_NONE,
                            torch.cuda.current_stream().cuda_stream)
    assert st == int(tg.Status.SCRATCH_LIMIT)
    assert tg.tl_status_string(st) == "TL_ERR_SCRATCH_LIMIT"
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())


def test_noalloc_takes_no_device_memory_after_its_first_call():
    """After the first call on the device, calls allocate nothing -- padded
    copies and split partial sums alike -- and every call's result is its own:
    stale partial sums or arrival counts left in the shared scratch by the
    previous call (same shape, other inputs) are never taken for this call's."""
    import tensor_core_gemm_tl_b200 as tg
    shapes = [(1000, 264, 2050, wl.F16, wl.EPI_BIAS_GELU, "pad_a split"),
              (1024, 1024, 2048, wl.BF16, wl.EPI_BIAS_GELU, "split")]
    runs = []
    for M, N, K, dt, epi, kind in shapes:
        for seed in (5, 6, 7):
            A, B, bias = wl.make_inputs(wl.custom("noalloc_mem", M, N, K, dt, epi), seed)
            bufs = _buffers(A, B, bias, dt)
            _check_plan_kind(_plan(M, N, K, dt, epi, bufs), kind)
            runs.append((bufs, dt, epi, _run(tg.tl_gemm, bufs, dt, epi)))
    _run(tg.tl_gemm_noalloc, runs[0][0], runs[0][1], runs[0][2])  # first call on the device: the set-up
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        for bufs, dt, epi, expected in runs:
            assert np.array_equal(_run(tg.tl_gemm_noalloc, bufs, dt, epi), expected)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
