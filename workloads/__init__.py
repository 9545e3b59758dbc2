"""Seeded synthetic inputs for the fused GEMM workloads.

This module is shared by the tests, the benchmark and the smoke check.  It
holds only the input recipe (shapes, distributions, seeds, rounding to the
16-bit input formats) and none of the GEMM's arithmetic: neither the oracle
nor the CUDA path lives here, and neither is imported from here.

Recipe (one numpy PCG64 stream per operand):
    A    <- default_rng(seed)      B <- default_rng(seed + 1)
    bias <- default_rng(seed + 2)
Values are drawn in float32 and rounded once, round-to-nearest-even, to fp16
(numpy's float16 cast) or bf16 (the upper half of the float32 pattern with
the discarded half rounded to nearest even).

The workloads are the pages' own GEMM -- 4096 x 4096 x 4096 in float16, from
"Designing High-Performance GPU Kernels with TileLang" (blog retelling),
section "performance comparison" and Step 4 -- plus the fused bias+GELU form
(TileLang GPU kernel design article, paragraph 5) at a small size, a
transformer MLP up-projection and a ragged / skinny set.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

F16, BF16 = 0, 1
EPI_NONE, EPI_BIAS_GELU, EPI_BIAS, EPI_GELU = 0, 1, 2, 3
EPI_BIAS_GELU_TANH, EPI_GELU_TANH = 4, 5
EPI_WITH_BIAS = (EPI_BIAS_GELU, EPI_BIAS, EPI_BIAS_GELU_TANH)
DTYPE_NAMES = {F16: "f16", BF16: "bf16"}


@dataclasses.dataclass(frozen=True)
class Dist:
    """A scalar distribution: 'uniform' on [-scale, scale] or 'normal' with std `scale`."""
    kind: str
    scale: float

    def describe(self) -> str:
        if self.kind == "uniform":
            return f"U[-{self.scale:g}, {self.scale:g}]"
        return f"N(0, std={self.scale:g})"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    K: int
    dtype: int
    epi: int
    a: Dist
    b: Dist
    bias: Optional[Dist]
    note: str = ""

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    def min_bytes(self) -> int:
        """Compulsory HBM bytes: read A and B once, write C once, read bias."""
        n = 2 * (self.M * self.K + self.K * self.N + self.M * self.N)
        if self.epi == EPI_BIAS_GELU:
            n += 2 * self.N
        return n

    def describe(self) -> dict:
        return {
            "workload": self.name, "M": self.M, "N": self.N, "K": self.K,
            "dtype": DTYPE_NAMES[self.dtype],
            "epilogue": "bias+gelu" if self.epi == EPI_BIAS_GELU else "none",
            "A": self.a.describe(), "B": self.b.describe(),
            "bias": self.bias.describe() if self.bias else None,
        }


def _u(s):
    return Dist("uniform", s)


def _n(s):
    return Dist("normal", s)


def _ragged(name, M, N, K, epi):
    s = 1.0 / np.sqrt(K)
    return Workload(name, M, N, K, BF16, epi, _n(s), _n(s), _n(0.1) if epi else None,
                    "A, B ~ N(0, 1/sqrt(K)) read as std 1/sqrt(K)")


WORKLOADS = {w.name: w for w in [
    Workload("gemm256_f16_bias_gelu", 256, 256, 256, F16, EPI_BIAS_GELU,
             _u(1.0), _u(1.0), _n(1.0)),
    Workload("gemm4096_f16", 4096, 4096, 4096, F16, EPI_NONE,
             _u(1.0 / 64), _u(1.0 / 64), None, "U[-1,1]/sqrt(K)"),
    Workload("gemm4096_f16_bias_gelu", 4096, 4096, 4096, F16, EPI_BIAS_GELU,
             _u(1.0 / 64), _u(1.0 / 64), _n(0.1), "U[-1,1]/sqrt(K)"),
    Workload("mlp_up_8192x16384x4096_bf16_bias_gelu", 8192, 16384, 4096, BF16, EPI_BIAS_GELU,
             _n(1.0), _n(1.0 / 64), _n(0.02), "B ~ N(0, 1/K) read as variance 1/K"),
    _ragged("ragged_4000x3000x2050_bf16", 4000, 3000, 2050, EPI_NONE),
    _ragged("ragged_4000x3000x2050_bf16_bias_gelu", 4000, 3000, 2050, EPI_BIAS_GELU),
    _ragged("tall_16384x1024x8192_bf16", 16384, 1024, 8192, EPI_NONE),
    _ragged("tall_16384x1024x8192_bf16_bias_gelu", 16384, 1024, 8192, EPI_BIAS_GELU),
    _ragged("skinny_128x16384x4096_bf16", 128, 16384, 4096, EPI_NONE),
    _ragged("skinny_128x16384x4096_bf16_bias_gelu", 128, 16384, 4096, EPI_BIAS_GELU),
]}

# The configuration the headline throughput is quoted on: the largest one, the
# MLP up-projection with the fused bias + GELU epilogue.
HEADLINE = "mlp_up_8192x16384x4096_bf16_bias_gelu"


def round_to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """float32 -> uint16 bit patterns of fp16 / bf16, round-to-nearest-even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    if dtype == BF16:
        u = x.view(np.uint32)
        # add 0x7fff plus the lsb of the kept half: ties go to the even pattern
        r = (u >> np.uint32(16)) & np.uint32(1)
        return ((u + np.uint32(0x7FFF) + r) >> np.uint32(16)).astype(np.uint16)
    raise ValueError(f"unknown dtype {dtype}")


def bits_to_float32(bits: np.ndarray, dtype: int) -> np.ndarray:
    """uint16 fp16 / bf16 bit patterns -> float32 (exact widening)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float32)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def draw(dist: Dist, shape, seed: int) -> np.ndarray:
    """float32 samples of `dist` from numpy PCG64 seeded with `seed`."""
    rng = np.random.default_rng(seed)
    n = int(np.prod(shape))
    if dist.kind == "uniform":
        x = rng.random(n, dtype=np.float32)
        x *= np.float32(2.0)
        x -= np.float32(1.0)
    elif dist.kind == "normal":
        x = rng.standard_normal(n, dtype=np.float32)
    else:
        raise ValueError(dist.kind)
    x *= np.float32(dist.scale)
    return x.reshape(shape)


def make_bias(w: Workload, seed: int = 0):
    """bias_bits (uint16, length N) for workload `w`, or None when its
    epilogue takes no bias."""
    return round_to_bits(draw(w.bias, (w.N,), seed + 2), w.dtype) if w.epi in EPI_WITH_BIAS else None


def make_inputs(w: Workload, seed: int = 0):
    """(A_bits, B_bits, bias_bits|None) for workload `w`, as uint16 arrays."""
    A = round_to_bits(draw(w.a, (w.M, w.K), seed), w.dtype)
    B = round_to_bits(draw(w.b, (w.K, w.N), seed + 1), w.dtype)
    return A, B, make_bias(w, seed)


def custom(name, M, N, K, dtype, epi, a=None, b=None, bias=None) -> Workload:
    """A workload of any shape with the given (or default unit-normal-ish) laws."""
    s = 1.0 / np.sqrt(max(K, 1))
    return Workload(name, M, N, K, dtype, epi, a or _u(1.0), b or _n(s),
                    (bias or _n(0.1)) if epi in EPI_WITH_BIAS else None)
