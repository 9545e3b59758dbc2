"""The checked build, libtlgemm_checked.so: the same sources compiled with
-DTL_CHECKED, whose kernels test their index invariants at run time (GEMM:
work items, tile coordinates, Tensor Memory columns, split-tile workspace
slabs; attention: Tensor Memory columns, key blocks, output rows; row
softmax: every bulk copy inside its row buffer and its row, 16-byte aligned)
and set bit 7 of the device error word on a violation instead of trapping.
On the CPU: it loads and exports the ABI.  On the GPU: parity cases covering
every configuration, split tiles, padding, element stores, B given
transposed and float32 C, attention of both head sizes and masks, and row
softmax through every kernel kind run through it against the oracle with no
check firing."""
import ctypes
import os
import re
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
import workloads as wl  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.path.join(ROOT, "tensor_core_gemm_tl_b200", "libtlgemm_checked.so")
HEADER = os.path.join(ROOT, "include", "tl_gemm.h")
ERR_CHECK = 128


def checked_lib():
    from tensor_core_gemm_tl_b200 import _binding
    assert os.path.exists(CHECKED), "libtlgemm_checked.so is missing: python tensor_core_gemm_tl_b200/build.py --checked"
    return _binding.load(CHECKED)


def test_checked_library_exports_the_abi():
    lib = checked_lib()
    names = sorted(set(re.findall(r"TL_API\s+[\w\s\*]+?\b(tl_\w+)\s*\(", open(HEADER).read())))
    for name in names:
        assert hasattr(lib, name), name
    assert lib.tl_num_configs() >= 3


CASES = [
    # (M, N, K, config, dtype, epilogue, B transposed, float32 C)
    (700, 900, 336, 1, wl.F16, wl.EPI_BIAS_GELU, False, False),
    (700, 900, 336, 2, wl.BF16, wl.EPI_NONE, True, False),
    (700, 900, 336, 3, wl.F16, wl.EPI_GELU_TANH, False, True),
    (700, 900, 336, 4, wl.BF16, wl.EPI_BIAS, False, False),
    (700, 900, 336, 5, wl.F16, wl.EPI_BIAS_GELU, True, False),
    (1024, 1024, 2048, 1, wl.BF16, wl.EPI_BIAS_GELU, False, False),   # split tail, single CTA
    (1024, 1280, 1536, 4, wl.F16, wl.EPI_BIAS_GELU, False, False),    # split tail, CTA pairs
    (1001, 999, 2051, 4, wl.BF16, wl.EPI_BIAS_GELU, False, False),    # padded A and B, element stores, split
    (300, 1001, 2050, 0, wl.BF16, wl.EPI_NONE, True, True),           # padded B^T, float32 element stores
    (4096, 4096, 4096, 0, wl.F16, wl.EPI_NONE, False, False),         # the timed shape
]


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,config,dt,epi,bt,f32", CASES)
def test_checked_kernel_no_invariant_fires(M, N, K, config, dt, epi, bt, f32):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gpu_util import accumulation_bound, compare, compare_f32, from_device, to_device
    import tensor_core_gemm_tl_b200 as tg
    lib = checked_lib()
    A, B, bias = wl.make_inputs(wl.custom("t", M, N, K, dt, epi), seed=M + K)
    dA = to_device(A, dt)
    dB = to_device(np.ascontiguousarray(B.T) if bt else B, dt)
    dbias = to_device(bias, dt) if bias is not None else None
    out = torch.empty((M, N), dtype=torch.float32 if f32 else (torch.float16 if dt == wl.F16 else torch.bfloat16),
                      device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    # the split tail taken wherever the last round is partial: its slots and
    # arrival words are among the checked invariants
    opt = tg.Options(config=config, b_layout=int(bt), c_float32=int(f32), force_split=int(config != 0))
    st = lib.tl_gemm_ex(dA.data_ptr(), dB.data_ptr(), dbias.data_ptr() if dbias is not None else None,
                        out.data_ptr(), M, N, K, dt, epi, stream or None, ctypes.byref(opt))
    assert st == 0
    word = ctypes.c_uint32(0)
    assert lib.tl_check_device(stream or None, ctypes.byref(word)) == 0, word.value
    assert not (word.value & ERR_CHECK)
    if M * N * K > 1 << 31:
        # the timed shape: sampled rows against the oracle
        rows = np.array([0, 1, 255, 256, 2047, 4095])
        ref = oracle.gemm(A, B, bias, dt, epi, rows=rows)
        C = from_device(out)[rows]
        compare(C, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref, rows=rows))
        return
    ref = oracle.gemm(A, B, bias, dt, epi)
    if f32:
        compare_f32(out.cpu().numpy(), ref, accumulation_bound(A, B, bias, dt, epi, ref, out_f32=True))
    else:
        compare(from_device(out), ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))


@pytest.mark.gpu
@pytest.mark.parametrize("D,causal,Sq,Sk", [(64, False, 300, 500), (128, True, 333, 333), (128, False, 1024, 4096)])
def test_checked_attention_no_invariant_fires(D, causal, Sq, Sk):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gpu_util import from_device, to_device
    lib = checked_lib()
    dt, B, H = wl.BF16, 1, 2
    rng = np.random.default_rng(D + Sq)
    Q, K, V = (wl.round_to_bits(rng.normal(size=(B, H, s, D)).astype(np.float32), dt) for s in (Sq, Sk, Sk))
    q, k, v = to_device(Q, dt), to_device(K, dt), to_device(V, dt)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream().cuda_stream
    scale = 1.0 / np.sqrt(D)
    st = lib.tl_attention_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), None, B, H, Sq, Sk, D,
                              dt, int(causal), ctypes.c_float(scale), stream or None)
    assert st == 0
    word = ctypes.c_uint32(0)
    assert lib.tl_check_device(stream or None, ctypes.byref(word)) == 0, word.value
    assert not (word.value & ERR_CHECK)
    ref, _ = oracle.attention(Q, K, V, dt, causal, scale)
    got = wl.bits_to_float32(from_device(out), dt).astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-2


@pytest.mark.gpu
@pytest.mark.parametrize("rows,cols,offset", [(64, 8192, 0), (37, 3000, 1), (9, 50257, 0), (5, 112000, 3)])
def test_checked_softmax_no_invariant_fires(rows, cols, offset):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gpu_util import from_device, to_device, ulp
    lib = checked_lib()
    dt = wl.BF16
    rng = np.random.default_rng(cols)
    X = wl.round_to_bits(rng.normal(size=(rows, cols)).astype(np.float32), dt)
    x = to_device(X, dt, offset)
    buf = torch.empty(x.numel() + offset, dtype=x.dtype, device="cuda")
    y = buf[offset:].view(x.shape)
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.tl_softmax_rows(x.data_ptr(), y.data_ptr(), rows, cols, dt, stream or None) == 0
    word = ctypes.c_uint32(0)
    assert lib.tl_check_device(stream or None, ctypes.byref(word)) == 0, word.value
    assert not (word.value & ERR_CHECK)
    ref = oracle.softmax_rows(X, dt)
    got = wl.bits_to_float32(from_device(y), dt).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 0.5 * ulp(ref, dt) + 1e-5 * ref + np.where(ref < 2.0 ** -126, ref, 0) + 1e-40)
