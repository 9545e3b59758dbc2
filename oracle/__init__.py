"""fp64 CPU oracle for C = epilogue(A . B) -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows); this
module only compiles it with gcc and marshals numpy arrays through ctypes.
Inputs are the raw 16-bit patterns of the fp16/bf16 operands; outputs are
float64 and are not rounded to the input dtype.

What it computes, and where that is stated:
  * "Designing High-Performance GPU Kernels with TileLang" (blog retelling),
    Step 4 "Tensor-Core GEMM": A (M x K) and B (K x N), row-major tiles,
    float32 accumulator -- here fp64, in which every fp16/bf16 product is
    exact.
  * TileLang GPU kernel design article, paragraph 5 (fused GEMM epilogue):
    bias add then GELU on the accumulator before the single store; bias is
    per column, GELU is the exact erf form (epilogues 1-3) or the tanh form
    of the GELU paper (epilogues 4, 5).
  * The same article, paragraph 6 (attention forward with online softmax,
    checked against PyTorch's scaled dot-product attention): the plain
    definition softmax(scale Q K^T) V, causal mask keeping key j <= query i.
  * The same article, paragraphs 5 and 3: a row softmax, and a float32 vector
    add (also the blog retelling, Step 3).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

F16 = 0
BF16 = 1
EPI_NONE = 0
EPI_BIAS_GELU = 1
EPI_BIAS = 2
EPI_GELU = 3
EPI_BIAS_GELU_TANH = 4
EPI_GELU_TANH = 5
EPI_WITH_BIAS = (EPI_BIAS_GELU, EPI_BIAS, EPI_BIAS_GELU_TANH)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# -ffp-contract=off keeps every multiply and add a separate IEEE fp64 step.
_CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile `src` (default oracle.c) into a shared library at `out` (gcc)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _bind(path):
    lib = ctypes.CDLL(path)
    i64, p = ctypes.c_int64, ctypes.c_void_p
    lib.oracle_gemm_rows.argtypes = [i64, i64, i64, p, p, p, ctypes.c_int, ctypes.c_int, p, i64, p]
    lib.oracle_gemm_rows.restype = ctypes.c_int
    lib.oracle_gemm.argtypes = [i64, i64, i64, p, p, p, ctypes.c_int, ctypes.c_int, p]
    lib.oracle_gemm.restype = ctypes.c_int
    lib.oracle_gemm_points.argtypes = [i64, i64, i64, p, p, p, ctypes.c_int, ctypes.c_int, p, p, i64, p]
    lib.oracle_gemm_points.restype = ctypes.c_int
    lib.oracle_decode_array.argtypes = [p, ctypes.c_int, p, i64]
    lib.oracle_decode_array.restype = None
    lib.oracle_gelu_array.argtypes = [p, p, i64]
    lib.oracle_gelu_array.restype = None
    lib.oracle_gelu_tanh_array.argtypes = [p, p, i64]
    lib.oracle_gelu_tanh_array.restype = None
    lib.oracle_attention_rows.argtypes = [i64, i64, i64, i64, p, p, p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_double, p, p, i64, p, p]
    lib.oracle_attention_rows.restype = ctypes.c_int
    lib.oracle_softmax_rows.argtypes = [i64, i64, p, ctypes.c_int, p]
    lib.oracle_softmax_rows.restype = ctypes.c_int
    lib.oracle_vector_add.argtypes = [i64, p, p, p]
    lib.oracle_vector_add.restype = None
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def _bits(x, name):
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError(f"{name}: expected the raw uint16 bit patterns, got {a.dtype}")
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data


def _check_shapes(A, B, bias, epi):
    if A.ndim != 2 or B.ndim != 2 or A.shape[1] != B.shape[0]:
        raise ValueError(f"shapes A{A.shape} B{B.shape} do not chain")
    if epi in EPI_WITH_BIAS:
        if bias is None or bias.shape != (B.shape[1],):
            raise ValueError("this epilogue needs a bias of length N")
    elif epi not in (EPI_NONE, EPI_GELU, EPI_GELU_TANH):
        raise ValueError(f"unknown epilogue {epi}")


class Oracle:
    """The oracle's entry points, bound to one compiled copy of the C source."""

    def __init__(self, lib):
        self._lib = lib

    def gemm(self, A, B, bias=None, dtype=F16, epi=EPI_NONE, rows=None) -> np.ndarray:
        """C (or the listed rows of C) in fp64. A, B, bias are uint16 bit arrays."""
        A, B = _bits(A, "A"), _bits(B, "B")
        bias = None if bias is None else _bits(bias, "bias")
        _check_shapes(A, B, bias, epi)
        M, K = A.shape
        N = B.shape[1]
        if rows is None:
            out = np.empty((M, N), np.float64)
            rc = self._lib.oracle_gemm(M, N, K, _ptr(A), _ptr(B), _ptr(bias), dtype, epi, _ptr(out))
        else:
            r = np.ascontiguousarray(rows, dtype=np.int64)
            out = np.empty((r.size, N), np.float64)
            rc = self._lib.oracle_gemm_rows(M, N, K, _ptr(A), _ptr(B), _ptr(bias), dtype, epi,
                                            _ptr(r), r.size, _ptr(out))
        if rc != 0:
            raise ValueError("oracle_gemm: bad row index or out of memory")
        return out

    def gemm_points(self, A, B, bias, dtype, epi, ii, jj) -> np.ndarray:
        """C[ii[p], jj[p]] in fp64 for each p, same summation order as gemm()."""
        A, B = _bits(A, "A"), _bits(B, "B")
        bias = None if bias is None else _bits(bias, "bias")
        _check_shapes(A, B, bias, epi)
        M, K = A.shape
        N = B.shape[1]
        ii = np.ascontiguousarray(ii, dtype=np.int64)
        jj = np.ascontiguousarray(jj, dtype=np.int64)
        if ii.shape != jj.shape:
            raise ValueError("ii and jj differ in shape")
        out = np.empty(ii.shape, np.float64)
        rc = self._lib.oracle_gemm_points(M, N, K, _ptr(A), _ptr(B), _ptr(bias), dtype, epi,
                                          _ptr(ii), _ptr(jj), ii.size, _ptr(out))
        if rc != 0:
            raise ValueError("oracle_gemm_points: index out of range")
        return out

    def decode(self, bits, dtype) -> np.ndarray:
        """fp16 / bf16 bit patterns -> float64 values, from the format definitions."""
        b = _bits(bits, "bits")
        out = np.empty(b.shape, np.float64)
        self._lib.oracle_decode_array(_ptr(b), dtype, _ptr(out), b.size)
        return out

    def gelu(self, x) -> np.ndarray:
        """Exact GELU x * Phi(x) in fp64, elementwise."""
        a = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty(a.shape, np.float64)
        self._lib.oracle_gelu_array(_ptr(a), _ptr(out), a.size)
        return out

    def gelu_tanh(self, x) -> np.ndarray:
        """Tanh-form GELU 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) in fp64."""
        a = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty(a.shape, np.float64)
        self._lib.oracle_gelu_tanh_array(_ptr(a), _ptr(out), a.size)
        return out

    def attention(self, Q, K, V, dtype, causal, scale, rows=None):
        """softmax(scale Q K^T [causal]) V in fp64 for Q (B, H, Sq, D), K and V
        (B, H, Sk, D) uint16 bit arrays.  Returns (O, lse): all of O (B, H, Sq, D)
        and lse (B, H, Sq), or, with rows = (bh_idx, q_idx) arrays, O (n, D) and
        lse (n,) for those (flattened batch*head, query) rows."""
        Q, K, V = _bits(Q, "Q"), _bits(K, "K"), _bits(V, "V")
        if Q.ndim != 4 or K.shape != V.shape or K.ndim != 4 or Q.shape[:2] != K.shape[:2] \
                or Q.shape[3] != K.shape[3]:
            raise ValueError(f"shapes Q{Q.shape} K{K.shape} V{V.shape} do not match")
        B, H, Sq, D = Q.shape
        Sk = K.shape[2]
        BH = B * H
        if rows is None:
            bh = np.repeat(np.arange(BH, dtype=np.int64), Sq)
            qi = np.tile(np.arange(Sq, dtype=np.int64), BH)
        else:
            bh = np.ascontiguousarray(rows[0], dtype=np.int64)
            qi = np.ascontiguousarray(rows[1], dtype=np.int64)
        O = np.empty((bh.size, D), np.float64)
        lse = np.empty(bh.size, np.float64)
        rc = self._lib.oracle_attention_rows(BH, Sq, Sk, D, _ptr(Q), _ptr(K), _ptr(V), dtype,
                                             int(bool(causal)), float(scale), _ptr(bh), _ptr(qi),
                                             bh.size, _ptr(O), _ptr(lse))
        if rc != 0:
            raise ValueError("oracle_attention_rows: bad index or size")
        if rows is None:
            return O.reshape(B, H, Sq, D), lse.reshape(B, H, Sq)
        return O, lse

    def softmax_rows(self, X, dtype) -> np.ndarray:
        """Row softmax of a (rows, cols) uint16 bit array, in fp64."""
        X = _bits(X, "X")
        if X.ndim != 2:
            raise ValueError("X must be 2-D")
        Y = np.empty(X.shape, np.float64)
        if self._lib.oracle_softmax_rows(X.shape[0], X.shape[1], _ptr(X), dtype, _ptr(Y)) != 0:
            raise ValueError("oracle_softmax_rows: bad size")
        return Y

    def vector_add(self, A, B) -> np.ndarray:
        """A + B for float32 vectors, each sum rounded once to float32."""
        A = np.ascontiguousarray(A, dtype=np.float32)
        B = np.ascontiguousarray(B, dtype=np.float32)
        if A.shape != B.shape:
            raise ValueError("shapes differ")
        C = np.empty_like(A)
        self._lib.oracle_vector_add(A.size, _ptr(A), _ptr(B), _ptr(C))
        return C

    def max_threads(self) -> int:
        """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
        return int(self._lib.oracle_max_threads())


_default = None


def _oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_load())
    return _default


def from_library(path: str) -> Oracle:
    """An Oracle bound to another build of the C source (tests plant mistakes this way)."""
    return Oracle(_bind(path))


def gemm(A, B, bias=None, dtype=F16, epi=EPI_NONE, rows=None) -> np.ndarray:
    """C (or the listed rows of C) in fp64. A, B, bias are uint16 bit arrays."""
    return _oracle().gemm(A, B, bias, dtype, epi, rows)


def gemm_points(A, B, bias, dtype, epi, ii, jj) -> np.ndarray:
    """C[ii[p], jj[p]] in fp64 for each p, same summation order as gemm()."""
    return _oracle().gemm_points(A, B, bias, dtype, epi, ii, jj)


def decode(bits, dtype) -> np.ndarray:
    """fp16 / bf16 bit patterns -> float64 values, from the format definitions."""
    return _oracle().decode(bits, dtype)


def gelu(x) -> np.ndarray:
    """Exact GELU x * Phi(x) in fp64, elementwise."""
    return _oracle().gelu(x)


def gelu_tanh(x) -> np.ndarray:
    """Tanh-form GELU in fp64, elementwise."""
    return _oracle().gelu_tanh(x)


def attention(Q, K, V, dtype, causal, scale, rows=None):
    """softmax(scale Q K^T [causal]) V and its log-sum-exp, in fp64."""
    return _oracle().attention(Q, K, V, dtype, causal, scale, rows)


def softmax_rows(X, dtype) -> np.ndarray:
    """Row softmax in fp64."""
    return _oracle().softmax_rows(X, dtype)


def vector_add(A, B) -> np.ndarray:
    """float32 A + B."""
    return _oracle().vector_add(A, B)


def max_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return _oracle().max_threads()
