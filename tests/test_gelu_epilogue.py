"""The epilogue's GELU: the kernel's float32 formula and constants checked on
the CPU against mpmath, and on the GPU the fused epilogue over every finite
fp16 and bf16 input value against the oracle."""
import os
import re
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import workloads as wl  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "tensor_core_gemm_tl_b200", "csrc", "gemm_kernel.cuh")


def kernel_constants():
    src = open(KERNEL).read()
    body = src[src.index("__device__ __forceinline__ float gelu_erf"):]
    body = body[:body.index("\n}\n")]
    m = re.search(r"constexpr float P_SQRT1_2 = ([0-9.eE+-]+)f \* ([0-9.eE+-]+)f;", body)
    p = np.float32(m.group(1)) * np.float32(m.group(2))          # folded at compile time in float
    cs = {int(k): float(v) for k, v in re.findall(r"C(\d) = ([0-9.eE+-]+)f", body)}
    nl = np.float32(re.search(r"NEG_HALF_LOG2E = ([0-9.eE+-]+)f;", body).group(1))
    return np.float32(p), [np.float32(cs[i]) for i in range(9)], nl


def gelu_like_kernel(x):
    """The kernel's float32 operation sequence, in numpy float32 (reciprocal and
    2^x taken correctly rounded here; the device's approximate ones add about
    2^-22 relative each)."""
    P, C, NL = kernel_constants()
    f = np.float32
    x = np.asarray(x, dtype=np.float32)
    a = np.minimum(np.abs(x), f(20))
    t = f(1) / (P * a + f(1))
    h = C[8] * t + C[7]
    for k in range(6, -1, -1):
        h = h * t + C[k]
    hi = a * a
    lo = (a.astype(np.float64) ** 2 - hi).astype(np.float32)
    e = np.exp2(hi * NL) * (f(1) - f(0.5) * lo)
    q = f(0.5) * h * e
    return x * np.where(x >= 0, f(1) - q, q)


def test_kernel_gelu_formula_accuracy():
    import mpmath as mp
    mp.mp.dps = 30
    xs = np.concatenate([np.linspace(-12, 12, 4801), np.geomspace(1e-20, 1, 200),
                         -np.geomspace(1e-20, 1, 200), [0.0, 25.0, -25.0, 1e30]]).astype(np.float32)
    got = gelu_like_kernel(xs).astype(np.float64)
    ref = np.array([float(mp.mpf(float(x)) * mp.ncdf(mp.mpf(float(x)))) for x in xs])
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-300)
    small = np.abs(xs) <= 9
    assert rel[small & (np.abs(ref) > 1e-37)].max() < 3e-6
    assert rel[np.abs(ref) > 1e-37].max() < 2e-5
    assert np.isnan(gelu_like_kernel(np.float32([np.nan]))[0])


@pytest.mark.gpu
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
def test_fused_gelu_every_finite_input(dt):
    """C = GELU(A.B + bias) with A.B = 0 and bias = every finite 16-bit value,
    so C[i, j] = GELU(bias[j]); compared with the oracle's fp64 GELU to half an
    output ulp plus 1e-5 relative (the kernel's float32 evaluation, device exp included)."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import oracle
    from gpu_util import run_library, ulp
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    expo = (allbits >> 10) & 0x1F if dt == wl.F16 else (allbits >> 7) & 0xFF
    finite = allbits[expo != (0x1F if dt == wl.F16 else 0xFF)]
    N, M, K = finite.size, 256, 16
    A = np.zeros((M, K), np.uint16)
    B = np.zeros((K, N), np.uint16)
    C = run_library(A, B, finite, dt, wl.EPI_BIAS_GELU)
    assert np.array_equal(C, np.repeat(C[:1], M, axis=0)), "rows differ"
    got = wl.bits_to_float32(C[0], dt).astype(np.float64)
    ref = oracle.gelu(oracle.decode(finite, dt))
    fin = np.isfinite(ref)
    assert np.all(np.isfinite(got[fin]))
    # the bf16 values whose GELU overflows fp32 (none) or whose fp64 GELU is NaN
    # (none for finite inputs) would show here
    err = np.abs(got[fin] - ref[fin])
    bound = 0.5 * ulp(np.abs(ref[fin]), dt) + 1e-5 * np.abs(ref[fin]) + 1e-45
    bad = err > bound
    assert not bad.any(), (wl.bits_to_float32(finite[fin][bad][:5], dt), got[fin][bad][:5], ref[fin][bad][:5])
