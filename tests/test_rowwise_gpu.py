"""Row softmax and vector add on the GPU (through the C ABI) against the
oracle.  Softmax: every element within half an output ulp plus 1e-5
relative (float32 evaluation with the hardware exp2) of the fp64 softmax;
probabilities below 2^-126 may come out as 0 (the flush-to-zero exp2), which
the bound allows by adding |ref| there.  Vector add: bit for bit."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
import workloads as wl  # noqa: E402
from gpu_util import from_device, to_device, ulp  # noqa: E402


def softmax_bound(ref, dt):
    """Half an output ulp + 1e-5 relative, and below 2^-126 the value itself."""
    return 0.5 * ulp(ref, dt) + 1e-5 * ref + np.where(ref < 2.0 ** -126, ref, 0.0) + 1e-40

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def run_softmax(X_bits, dt, offset=0, y_offset=None):
    import tensor_core_gemm_tl_b200 as tg
    x = to_device(X_bits, dt, offset)
    y_offset = offset if y_offset is None else y_offset
    if y_offset:
        buf = torch.empty(x.numel() + y_offset, dtype=x.dtype, device="cuda")
        y = buf[y_offset:].view(x.shape)
    else:
        y = torch.empty_like(x)
    tg.softmax(x, out=y)
    torch.cuda.synchronize()
    return from_device(y)


@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 7), (64, 33), (333, 64), (1001, 100), (1000, 128),
                                       (1000, 256), (257, 1000), (128, 1024), (40, 1025), (17, 4096),
                                       (9, 12288), (11, 16385), (8, 50000), (3, 50257), (5, 112000),
                                       (2, 200000)])
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
def test_softmax_vs_oracle(rows, cols, dt):
    rng = np.random.default_rng(rows * 7 + cols)
    X = wl.round_to_bits((rng.normal(size=(rows, cols)) * 3).astype(np.float32), dt)
    ref = oracle.softmax_rows(X, dt)
    Y = wl.bits_to_float32(run_softmax(X, dt), dt).astype(np.float64)
    bound = softmax_bound(ref, dt)
    assert np.all(np.abs(Y - ref) <= bound), np.max(np.abs(Y - ref) - bound)


@pytest.mark.parametrize("rows,cols", [(16384, 8192), (4096, 50257), (262144, 128)])
def test_softmax_benchmark_sizes_sampled_rows(rows, cols):
    """The timed shapes, computed whole on the GPU; sampled rows (first, last
    and random) checked against the oracle."""
    dt = wl.BF16
    rng = np.random.default_rng(cols)
    X = wl.round_to_bits(rng.normal(size=(rows, cols)).astype(np.float32), dt)
    Y = run_softmax(X, dt)
    pick = np.unique(np.concatenate([[0, rows - 1], rng.integers(0, rows, 200)]))
    ref = oracle.softmax_rows(np.ascontiguousarray(X[pick]), dt)
    got = wl.bits_to_float32(Y[pick], dt).astype(np.float64)
    assert np.all(np.abs(got - ref) <= softmax_bound(ref, dt))


@pytest.mark.parametrize("offset", [1, 3])
def test_softmax_unaligned(offset):
    dt = wl.BF16
    rng = np.random.default_rng(offset)
    for rows, cols in ((10, 512), (5, 3000)):
        X = wl.round_to_bits(rng.normal(size=(rows, cols)).astype(np.float32), dt)
        ref = oracle.softmax_rows(X, dt)
        Y = wl.bits_to_float32(run_softmax(X, dt, offset), dt).astype(np.float64)
        assert np.all(np.abs(Y - ref) <= softmax_bound(ref, dt))


@pytest.mark.parametrize("x_off,y_off", [(1, 2), (0, 3), (5, 0)])
@pytest.mark.parametrize("cols", [600, 3000, 20001, 70000])
def test_softmax_input_and_output_differently_aligned(x_off, y_off, cols):
    """X and Y at different distances from a 16-byte boundary: no row body can
    move as whole words on both sides (element path throughout)."""
    dt = wl.F16
    rng = np.random.default_rng(cols + x_off)
    X = wl.round_to_bits(rng.normal(size=(6, cols)).astype(np.float32), dt)
    ref = oracle.softmax_rows(X, dt)
    Y = wl.bits_to_float32(run_softmax(X, dt, x_off, y_off), dt).astype(np.float64)
    assert np.all(np.abs(Y - ref) <= softmax_bound(ref, dt))


def test_softmax_constant_and_dominant_rows():
    dt = wl.F16
    X = np.zeros((4, 777), np.float32)
    X[1, :] = -3.0
    X[2, 100] = 30000.0
    X[3, :] = -60000.0
    X[3, 5] = 0.0
    Y = wl.bits_to_float32(run_softmax(wl.round_to_bits(X, dt), dt), dt).astype(np.float64)
    one_over = float(wl.bits_to_float32(wl.round_to_bits(np.float32([1 / 777]), dt), dt)[0])
    assert np.all(Y[0] == one_over) and np.all(Y[1] == one_over)
    assert Y[2, 100] == 1.0 and np.count_nonzero(Y[2]) == 1
    assert Y[3, 5] == 1.0 and np.count_nonzero(Y[3]) == 1


@pytest.mark.parametrize("n", [1, 3, 4, 1000003, 1 << 24])
@pytest.mark.parametrize("offset", [0, 1])
def test_vector_add_bit_exact(n, offset):
    import tensor_core_gemm_tl_b200 as tg
    rng = np.random.default_rng(n + offset)
    A = (rng.normal(size=n) * 1e3).astype(np.float32)
    B = (rng.normal(size=n)).astype(np.float32)
    a = torch.from_numpy(np.concatenate([np.zeros(offset, np.float32), A])).cuda()[offset:]
    b = torch.from_numpy(B).cuda()
    c = tg.vector_add(a, b)
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy(), oracle.vector_add(A, B))
