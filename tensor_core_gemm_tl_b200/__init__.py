"""B200-native (sm_100a) fused tensor-core GEMM:  C = epilogue(A . B).

The work runs in libtlgemm.so (hand-written tcgen05 / TMA kernels behind a C
ABI, include/tl_gemm.h).  This package is its Python binding: the raw C-ABI
calls (``tl_gemm``, ``tl_gemm_ex``, ``tl_check_device``, ``tl_gemm_plan`` ...)
on device pointers, and ``gemm`` which takes torch CUDA tensors and passes
their pointers and the current stream.  PyTorch only provides device memory
and streams; nothing here computes.

Importing the package fails if the library is not built -- there is no CPU
or library fallback.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    LIB_PATH, Options, Plan, Status, TLError, TL_BF16, TL_EPI_BIAS, TL_EPI_BIAS_GELU, TL_EPI_GELU,
    TL_EPI_NONE, TL_EPI_BIAS_GELU_TANH, TL_EPI_GELU_TANH, TL_EPI_WITH_BIAS, TL_F16,
    SIGNATURES, tl_attention_fwd, tl_check_device, tl_config_name, tl_gemm, tl_gemm_ex, tl_gemm_noalloc,
    tl_gemm_plan, tl_num_configs, tl_softmax_rows, tl_vector_add,
    tl_status_string, tl_version,
)

__all__ = [
    "gemm", "attention", "softmax", "vector_add", "check_device", "plan", "configs", "tl_attention_fwd",
    "tl_softmax_rows", "tl_vector_add", "Options", "Plan", "Status", "TLError",
    "tl_gemm", "tl_gemm_ex", "tl_gemm_noalloc", "tl_check_device", "tl_gemm_plan", "tl_num_configs", "tl_config_name",
    "tl_status_string", "tl_version", "TL_F16", "TL_BF16", "TL_EPI_NONE", "TL_EPI_BIAS_GELU",
    "TL_EPI_BIAS", "TL_EPI_GELU", "TL_EPI_BIAS_GELU_TANH", "TL_EPI_GELU_TANH",
]


def _dtype_code(t):
    import torch
    if t.dtype == torch.float16:
        return TL_F16
    if t.dtype == torch.bfloat16:
        return TL_BF16
    raise TypeError(f"expected float16 or bfloat16, got {t.dtype}")


_EPILOGUES = {None: TL_EPI_NONE, "none": TL_EPI_NONE, "bias_gelu": TL_EPI_BIAS_GELU,
              "bias+gelu": TL_EPI_BIAS_GELU, "bias": TL_EPI_BIAS, "gelu": TL_EPI_GELU,
              "bias_gelu_tanh": TL_EPI_BIAS_GELU_TANH, "gelu_tanh": TL_EPI_GELU_TANH}


def _require_device_tensor(name, t, device, dtype=None, shape=None):
    """Raise ValueError unless `t` is a contiguous CUDA tensor on `device` (and
    of `dtype` / `shape` when given): a host or foreign-device pointer must
    never reach a kernel's loads or stores."""
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _epi_code(epilogue):
    if isinstance(epilogue, int) and TL_EPI_NONE <= epilogue <= TL_EPI_GELU_TANH:
        return epilogue
    if epilogue in _EPILOGUES:
        return _EPILOGUES[epilogue]
    raise ValueError(f"unknown epilogue {epilogue!r}")


def gemm(A, B, bias=None, epilogue=None, out=None, stream=None, config: int = 0, timeout_ns: int = 0,
         no_split: bool = False, b_transposed: bool = False, out_dtype=None, raster_group: int = 0,
         force_split: bool = False):
    """C = epilogue(A @ B) for row-major CUDA tensors A (M x K) and B (K x N),
    or B given as N x K (``b_transposed=True``: C = epilogue(A @ B.T), the
    layout of a linear layer's weight).

    ``epilogue`` is None / "none", "bias_gelu", "bias", "gelu",
    "bias_gelu_tanh" or "gelu_tanh" (``bias`` of length N for the ones that
    name it; default "bias_gelu" when a bias is given).  C has A's dtype, or
    float32 with ``out_dtype=torch.float32`` (or a float32 ``out``): the
    epilogue's fp32 result without rounding to 16 bits.  ``out`` (M x N) is
    written if given, else allocated.  Runs asynchronously on ``stream``
    (default: torch's current stream).  ``config`` = k > 0 forces kernel
    configuration k - 1; ``raster_group`` > 0 sets the output-tile rows per
    rasterisation group.
    """
    import torch
    epi = _epi_code(epilogue if epilogue is not None else ("bias_gelu" if bias is not None else None))
    k_of_b = B.shape[1] if (b_transposed and B.dim() == 2) else (B.shape[0] if B.dim() == 2 else None)
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != k_of_b:
        raise ValueError(f"shapes {tuple(A.shape)} and {tuple(B.shape)} do not chain")
    for name, t in (("A", A), ("B", B)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if B.device != A.device:
        raise ValueError(f"B is on {B.device}, A on {A.device}")
    dt = _dtype_code(A)
    if B.dtype != A.dtype:
        raise TypeError("A and B must have the same dtype")
    M, K = A.shape
    N = B.shape[0] if b_transposed else B.shape[1]
    if epi in TL_EPI_WITH_BIAS:
        if bias is None:
            raise ValueError("this epilogue needs a contiguous CUDA bias of length N in the input dtype")
        _require_device_tensor("bias", bias, A.device, A.dtype, (N,))
    if out_dtype is None:
        out_dtype = out.dtype if out is not None else A.dtype
    if out_dtype not in (A.dtype, torch.float32):
        raise TypeError("C is either A's dtype or float32")
    c_f32 = out_dtype == torch.float32
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A.device)
    else:
        _require_device_tensor("out", out, A.device, out_dtype, (M, N))
    s = stream if stream is not None else torch.cuda.current_stream(A.device)
    bias_ptr = bias.data_ptr() if bias is not None and epi in TL_EPI_WITH_BIAS else 0
    with torch.cuda.device(A.device):
        if config or timeout_ns or no_split or b_transposed or c_f32 or raster_group or force_split:
            opt = Options(config=config, inject_fault=0, timeout_ns=timeout_ns, no_split=int(no_split),
                          b_layout=int(bool(b_transposed)), c_float32=int(c_f32), raster_group=raster_group,
                          force_split=int(bool(force_split)))
            st = tl_gemm_ex(A.data_ptr(), B.data_ptr(), bias_ptr, out.data_ptr(), M, N, K, dt, epi,
                            s.cuda_stream, opt)
        else:
            st = tl_gemm(A.data_ptr(), B.data_ptr(), bias_ptr, out.data_ptr(), M, N, K, dt, epi, s.cuda_stream)
    if st != 0:
        raise TLError(st, "tl_gemm")
    return out


def attention(q, k, v, causal: bool = False, scale: float = 0.0, out=None, lse=None, stream=None):
    """softmax(scale q k^T [causal]) v for CUDA tensors q (B, H, Sq, D) and
    k, v (B, H, Sk, D), fp16 or bf16, D in {64, 128}; scale 0 = 1/sqrt(D).
    Returns out (B, H, Sq, D); fills `lse` (B, H, Sq) float32 if given."""
    import torch
    if q.dim() != 4 or k.shape != v.shape or k.dim() != 4 or q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3]:
        raise ValueError(f"shapes q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)} do not match")
    if not q.is_cuda:
        raise ValueError("q must be a CUDA tensor")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_device_tensor(name, t, q.device, q.dtype)
    dt = _dtype_code(q)
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    # every given tensor is checked before anything is allocated
    if lse is not None:
        _require_device_tensor("lse", lse, q.device, torch.float32, (B, H, Sq))
    if out is None:
        out = torch.empty_like(q)
    else:
        _require_device_tensor("out", out, q.device, q.dtype, q.shape)
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        st = tl_attention_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                              lse.data_ptr() if lse is not None else 0, B, H, Sq, Sk, D, dt, causal, scale,
                              s.cuda_stream)
    if st != 0:
        raise TLError(st, "tl_attention_fwd")
    return out


def softmax(x, out=None, stream=None):
    """Row softmax of a contiguous 2-D fp16/bf16 CUDA tensor (over the last dim)."""
    import torch
    if x.dim() != 2 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D CUDA tensor")
    dt = _dtype_code(x)
    if out is None:
        out = torch.empty_like(x)
    else:
        _require_device_tensor("out", out, x.device, x.dtype, x.shape)
    s = stream if stream is not None else torch.cuda.current_stream(x.device)
    with torch.cuda.device(x.device):
        st = tl_softmax_rows(x.data_ptr(), out.data_ptr(), x.shape[0], x.shape[1], dt, s.cuda_stream)
    if st != 0:
        raise TLError(st, "tl_softmax_rows")
    return out


def vector_add(a, b, out=None, stream=None):
    """a + b for contiguous float32 CUDA tensors of one shape."""
    import torch
    if not a.is_cuda:
        raise ValueError("a must be a CUDA tensor")
    _require_device_tensor("a", a, a.device, torch.float32)
    _require_device_tensor("b", b, a.device, torch.float32, a.shape)
    if out is None:
        out = torch.empty_like(a)
    else:
        _require_device_tensor("out", out, a.device, torch.float32, a.shape)
    s = stream if stream is not None else torch.cuda.current_stream(a.device)
    with torch.cuda.device(a.device):
        st = tl_vector_add(a.data_ptr(), b.data_ptr(), out.data_ptr(), a.numel(), s.cuda_stream)
    if st != 0:
        raise TLError(st, "tl_vector_add")
    return out


def check_device(stream=None) -> int:
    """Synchronize and return the device error word (0 = no wait ran out)."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    st, word = tl_check_device(s.cuda_stream)
    if st not in (0, int(Status.DEVICE_TIMEOUT)):
        raise TLError(st, "tl_check_device")
    return word


def plan(M, N, K, dtype=TL_F16, epilogue=None, num_sms=148, config=0, ptrs=(256, 256, 256, 256),
         b_transposed=False, no_split=False, c_float32=False, force_split=False, raster_group=0) -> dict:
    """The host plan for a call (no GPU needed): config, grid, padding, store path."""
    a, b, bias, c = ptrs
    epi = _epi_code(epilogue)
    opt = Options(config=config, b_layout=int(b_transposed), no_split=int(no_split), c_float32=int(c_float32),
                  force_split=int(force_split), raster_group=raster_group) \
        if (config or b_transposed or no_split or c_float32 or force_split or raster_group) else None
    st, p = tl_gemm_plan(a, b, bias if epi in TL_EPI_WITH_BIAS else 0, c, M, N, K, dtype, epi, num_sms, opt)
    if st != 0:
        raise TLError(st, "tl_gemm_plan")
    d = p.as_dict()
    d["config_name"] = tl_config_name(d["config"])
    return d


def configs() -> list[str]:
    return [tl_config_name(i) for i in range(tl_num_configs())]
