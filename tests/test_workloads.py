"""The seeded input generator: rounding against torch's casts, determinism,
and that each workload draws the law it states."""
import numpy as np
import pytest
import torch

import workloads as wl


def _ties_and_randoms(rng, n):
    x = rng.normal(0, 3, n).astype(np.float32)
    # exact ties for bf16: low half 0x8000 with both parities of the kept lsb
    u = rng.integers(0x3F000000, 0x40800000, n // 4, dtype=np.uint32)
    ties = ((u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    return np.concatenate([x, ties, np.float32([0.0, -0.0, 1e-40, -3e-39, 65504.0, 1e-8])])


@pytest.mark.parametrize("dtype,tdt", [(wl.F16, torch.float16), (wl.BF16, torch.bfloat16)])
def test_round_to_bits_matches_torch(dtype, tdt):
    x = _ties_and_randoms(np.random.default_rng(0), 20000)
    got = wl.round_to_bits(x, dtype)
    ref = torch.from_numpy(x).to(tdt).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    back = wl.bits_to_float32(got, dtype)
    assert np.array_equal(back, torch.from_numpy(x).to(tdt).float().numpy())


def test_make_inputs_is_deterministic_and_streams_differ():
    w = wl.custom("t", 64, 48, 32, wl.BF16, wl.EPI_BIAS_GELU)
    a1, b1, c1 = wl.make_inputs(w, seed=5)
    a2, b2, c2 = wl.make_inputs(w, seed=5)
    assert np.array_equal(a1, a2) and np.array_equal(b1, b2) and np.array_equal(c1, c2)
    a3, _, _ = wl.make_inputs(w, seed=6)
    assert not np.array_equal(a1, a3)
    assert a1.shape == (64, 32) and b1.shape == (32, 48) and c1.shape == (48,)


def test_epilogue_free_workload_has_no_bias():
    w = wl.WORKLOADS["gemm4096_f16"]
    assert w.bias is None and w.epi == wl.EPI_NONE


@pytest.mark.parametrize("name", ["gemm256_f16_bias_gelu", "ragged_4000x3000x2050_bf16_bias_gelu"])
def test_workload_laws(name):
    w = wl.WORKLOADS[name]
    A, B, bias = wl.make_inputs(w, 0)
    for bits, d in ((A, w.a), (B, w.b), (bias, w.bias)):
        v = wl.bits_to_float32(bits, w.dtype).astype(np.float64)
        if d.kind == "uniform":
            assert v.min() >= -d.scale and v.max() <= d.scale
            assert abs(v.std() - d.scale / np.sqrt(3)) < 0.05 * d.scale
        else:
            assert abs(v.std() - d.scale) < 0.1 * d.scale
        assert abs(v.mean()) < 0.1 * d.scale + 0.1 * d.scale


def test_table_of_workloads():
    names = set(wl.WORKLOADS)
    assert wl.HEADLINE in names
    shapes = {(w.M, w.N, w.K) for w in wl.WORKLOADS.values()}
    assert {(256, 256, 256), (4096, 4096, 4096), (8192, 16384, 4096), (4000, 3000, 2050),
            (16384, 1024, 8192), (128, 16384, 4096)} <= shapes
    for w in wl.WORKLOADS.values():
        assert w.flops == 2 * w.M * w.N * w.K


def test_test_side_rounding_matches_torch():
    """The tests' fp64 -> fp16/bf16 rounding (used for ulp diagnostics) agrees
    with torch's casts on float32-representable inputs."""
    import sys, os
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from gpu_util import round_to_dtype
    x = _ties_and_randoms(np.random.default_rng(3), 4000)
    x = x[np.abs(x) < 60000]
    for dt, tdt in ((wl.F16, torch.float16), (wl.BF16, torch.bfloat16)):
        ref = torch.from_numpy(x).to(tdt).double().numpy()
        assert np.array_equal(round_to_dtype(x.astype(np.float64), dt), ref)
