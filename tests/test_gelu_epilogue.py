"""The epilogue's GELU (exact erf form and tanh form): the kernel's float32
formulas and constants checked on the CPU against mpmath, and on the GPU the
fused epilogue over every finite fp16 and bf16 input value against the
oracle, with 16-bit and with float32 output."""
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
    body = src[src.index("__device__ __forceinline__ float2 gelu_erf2"):]
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


def kernel_tanh_constant():
    src = open(KERNEL).read()
    body = src[src.index("__device__ __forceinline__ float2 gelu_tanh2"):]
    body = body[:body.index("\n}\n")]
    k0 = np.float32(re.search(r"constexpr float K0 = ([0-9.eE+-]+)f;", body).group(1))
    k1c = np.float32(re.search(r"constexpr float K1 = ([0-9.eE+-]+)f \* K0;", body).group(1))
    return k0, np.float32(k1c * k0)


def gelu_tanh_like_kernel(x):
    """The kernel's float32 tanh-GELU sequence in numpy float32 (2^x and the
    reciprocal correctly rounded here; the device's add about 2^-22 each)."""
    K0, K1 = kernel_tanh_constant()
    f = np.float32
    x = np.asarray(x, dtype=np.float32)
    with np.errstate(over="ignore", under="ignore"):
        # fmaf(K1, x * x, K0): one rounding of the exact K1 x^2 + K0
        a = np.abs(x) * (np.float64(K1) * (x * x).astype(np.float64) + np.float64(K0)).astype(np.float32)
        e = np.exp2(-a.astype(np.float64)).astype(np.float32)
        s = (1.0 / (f(1) + e).astype(np.float64)).astype(np.float32)
        return x * np.where(x >= 0, s, e * s)


def tanh_rel_bound(x):
    """Relative error allowed for the float32 tanh GELU at x: the rounding of
    a = |2u| log2(e) (about 2 ulps) carried through 2^-a, plus the device's
    approximate 2^x and reciprocal."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x) * (2.3022082 + 0.10294 * x * x)
    return 1e-6 + 2.5e-7 * a


def _mp_gelu_tanh(x):
    import mpmath as mp
    # for x < 0, 1 + tanh(u) loses about 0.87 |u| digits: carry that many more
    u = abs(0.7978845608028654 * (x + 0.044715 * x ** 3)) if x < 0 else 0.0
    with mp.workdps(30 + int(0.87 * u)):
        xm = mp.mpf(x)
        return float(xm / 2 * (1 + mp.tanh(mp.sqrt(2 / mp.pi) * (xm + mp.mpf("0.044715") * xm ** 3))))


def test_kernel_gelu_tanh_formula_accuracy():
    import mpmath as mp
    mp.mp.dps = 30
    xs = np.concatenate([np.linspace(-12, 12, 4801), np.geomspace(1e-20, 1, 200),
                         -np.geomspace(1e-20, 1, 200), [0.0, 25.0, -25.0, 1e30]]).astype(np.float32)
    got = gelu_tanh_like_kernel(xs).astype(np.float64)
    ref = np.array([_mp_gelu_tanh(float(x)) for x in xs])
    keep = np.abs(ref) > 1e-37
    rel = np.abs(got - ref)[keep] / np.abs(ref[keep])
    assert np.all(rel < tanh_rel_bound(xs[keep]) - 5e-7), rel.max()  # room for the device's MUFU ops
    assert np.isnan(gelu_tanh_like_kernel(np.float32([np.nan]))[0])


def _finite_patterns(dt):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    expo = (allbits >> 10) & 0x1F if dt == wl.F16 else (allbits >> 7) & 0xFF
    return allbits[expo != (0x1F if dt == wl.F16 else 0xFF)]


@pytest.mark.gpu
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
@pytest.mark.parametrize("form", ["erf", "tanh"])
@pytest.mark.parametrize("out_f32", [False, True])
def test_fused_gelu_forms_every_finite_input(dt, form, out_f32):
    """Both GELU forms, 16-bit and float32 output: C = GELU(0 + bias) for bias
    = every finite 16-bit value, against the oracle's fp64 GELU."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import oracle
    from gpu_util import F32, run_library, ulp
    finite = _finite_patterns(dt)
    N, M, K = finite.size, 256, 16
    A = np.zeros((M, K), np.uint16)
    B = np.zeros((K, N), np.uint16)
    epi = wl.EPI_BIAS_GELU if form == "erf" else wl.EPI_BIAS_GELU_TANH
    C = run_library(A, B, finite, dt, epi, out_f32=out_f32)
    assert np.array_equal(C, np.repeat(C[:1], M, axis=0)), "rows differ"
    got = C[0].astype(np.float64) if out_f32 else wl.bits_to_float32(C[0], dt).astype(np.float64)
    x = oracle.decode(finite, dt)
    ref = oracle.gelu(x) if form == "erf" else oracle.gelu_tanh(x)
    assert np.all(np.isfinite(got))
    if form == "erf":
        rel = np.where(np.abs(x) <= 9, 4e-6, 2e-5)
    else:
        rel = tanh_rel_bound(x)
    # a result below the smallest normal float32 (2^-126) has fewer significant
    # bits, and so do the kernel's intermediates on the way to it: the relative
    # allowance applies to max(|ref|, 2^-126) there
    bound = 0.5 * ulp(np.abs(ref), F32 if out_f32 else dt) + rel * np.maximum(np.abs(ref), 2.0 ** -126) + 1e-45
    bad = np.abs(got - ref) > bound
    assert not bad.any(), (x[bad][:5], got[bad][:5], ref[bad][:5])


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
