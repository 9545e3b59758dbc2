"""ctypes binding of libtlgemm.so: the C-ABI calls under the same names.

Argument marshalling only -- every step of the GEMM runs in the library's CUDA
kernels.  There is no fallback: if the library is missing or cannot be loaded,
importing the package raises.
"""
from __future__ import annotations

import ctypes
import enum
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtlgemm.so")

TL_F16, TL_BF16 = 0, 1
TL_EPI_NONE, TL_EPI_BIAS_GELU, TL_EPI_BIAS, TL_EPI_GELU = 0, 1, 2, 3
TL_EPI_BIAS_GELU_TANH, TL_EPI_GELU_TANH = 4, 5
TL_EPI_WITH_BIAS = (TL_EPI_BIAS_GELU, TL_EPI_BIAS, TL_EPI_BIAS_GELU_TANH)


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = 1
    UNSUPPORTED = 2
    MISALIGNED = 3
    CUDA = 4
    DEVICE_TIMEOUT = 5
    SCRATCH_LIMIT = 6


class TLError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = Status(status)
        super().__init__(f"{what}: {self.status.name}" if what else self.status.name)


class Options(ctypes.Structure):
    """tl_gemm_options: config (0 = library's choice, k = configuration k-1),
    inject_fault (test hook: 1 device-side stall, 2 host-side encode failure), timeout_ns (0 = 10 s), no_split (1 = never split
    the tiles of a short last round), b_layout (1 = B given as N x K),
    c_float32 (1 = C is float32), raster_group (tile rows per rasterisation
    group, 0 = library's choice), force_split (1 = cut a partial last round
    along K whenever possible)."""
    _fields_ = [("config", ctypes.c_int32), ("inject_fault", ctypes.c_int32),
                ("timeout_ns", ctypes.c_uint64), ("no_split", ctypes.c_int32), ("b_layout", ctypes.c_int32),
                ("c_float32", ctypes.c_int32), ("raster_group", ctypes.c_int32), ("force_split", ctypes.c_int32)]


class Plan(ctypes.Structure):
    """tl_plan: the host-side decision for one call."""
    _fields_ = [("config", ctypes.c_int32), ("block_m", ctypes.c_int32), ("block_n", ctypes.c_int32),
                ("block_k", ctypes.c_int32), ("stages", ctypes.c_int32), ("tiles_m", ctypes.c_int32),
                ("tiles_n", ctypes.c_int32), ("grid", ctypes.c_int32), ("cluster_ctas", ctypes.c_int32),
                ("split", ctypes.c_int32), ("full_tiles", ctypes.c_int32), ("pad_a", ctypes.c_int32),
                ("pad_b", ctypes.c_int32), ("direct_store", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("workspace_bytes", ctypes.c_int64),
                ("tail_units", ctypes.c_int32), ("num_slots", ctypes.c_int32),
                ("raster_group", ctypes.c_int32), ("reserved", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


# name -> (restype, argtypes); every symbol include/tl_gemm.h declares
_P, _I64, _I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
SIGNATURES = {
    "tl_gemm": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, _P]),
    "tl_gemm_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, _P]),
    "tl_gemm_ex": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, _P,
                                  ctypes.POINTER(Options)]),
    "tl_check_device": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "tl_softmax_rows": (ctypes.c_int, [_P, _P, _I64, _I64, ctypes.c_int, _P]),
    "tl_vector_add": (ctypes.c_int, [_P, _P, _P, _I64, _P]),
    "tl_attention_fwd": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, _I32,
                                        ctypes.c_float, _P]),
    "tl_gemm_plan": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, _I32,
                                    ctypes.POINTER(Options), ctypes.POINTER(Plan)]),
    "tl_num_configs": (_I32, []),
    "tl_config_name": (ctypes.c_char_p, [_I32]),
    "tl_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "tl_version": (_I32, []),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python tensor_core_gemm_tl_b200/build.py`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load()


def _check(st: int, what: str) -> None:
    if st != 0:
        raise TLError(st, what)


def tl_gemm(A: int, B: int, bias: int | None, C: int, M: int, N: int, K: int, dtype: int, epi: int,
            stream: int = 0) -> int:
    """C = epilogue(A.B) on device pointers; returns the tl_status code."""
    return _lib.tl_gemm(A, B, bias or None, C, M, N, K, dtype, epi, stream or None)


def tl_gemm_noalloc(A: int, B: int, bias: int | None, C: int, M: int, N: int, K: int, dtype: int, epi: int,
                    stream: int = 0) -> int:
    """tl_gemm without any allocation: padded operand copies go to the library's
    fixed scratch area; returns the tl_status code (SCRATCH_LIMIT if too big)."""
    return _lib.tl_gemm_noalloc(A, B, bias or None, C, M, N, K, dtype, epi, stream or None)


def tl_gemm_ex(A, B, bias, C, M, N, K, dtype, epi, stream=0, options: Options | None = None) -> int:
    return _lib.tl_gemm_ex(A, B, bias or None, C, M, N, K, dtype, epi, stream or None,
                           ctypes.byref(options) if options is not None else None)


def tl_attention_fwd(Q, K, V, O, lse, batch, heads, seq_q, seq_k, head_dim, dtype, causal, softmax_scale,
                     stream=0) -> int:
    """Attention forward on device pointers; returns the tl_status code."""
    return _lib.tl_attention_fwd(Q, K, V, O, lse or None, batch, heads, seq_q, seq_k, head_dim, dtype,
                                 int(bool(causal)), float(softmax_scale), stream or None)


def tl_softmax_rows(X, Y, rows, cols, dtype, stream=0) -> int:
    return _lib.tl_softmax_rows(X, Y, rows, cols, dtype, stream or None)


def tl_vector_add(A, B, C, n, stream=0) -> int:
    return _lib.tl_vector_add(A, B, C, n, stream or None)


def tl_check_device(stream: int = 0) -> tuple[int, int]:
    """(status, raw device error word) after synchronizing `stream`."""
    detail = ctypes.c_uint32(0)
    st = _lib.tl_check_device(stream or None, ctypes.byref(detail))
    return st, detail.value


def tl_gemm_plan(A, B, bias, C, M, N, K, dtype, epi, num_sms=0, options: Options | None = None):
    """(status, Plan) -- the decision tl_gemm takes, without a launch."""
    plan = Plan()
    st = _lib.tl_gemm_plan(A, B, bias or None, C, M, N, K, dtype, epi, num_sms,
                           ctypes.byref(options) if options is not None else None, ctypes.byref(plan))
    return st, plan


def tl_num_configs() -> int:
    return _lib.tl_num_configs()


def tl_config_name(i: int) -> str | None:
    r = _lib.tl_config_name(i)
    return r.decode() if r is not None else None


def tl_status_string(s: int) -> str:
    return _lib.tl_status_string(s).decode()


def tl_version() -> int:
    return _lib.tl_version()
