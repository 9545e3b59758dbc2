"""Helpers shared by the GPU parity tests: move seeded bit arrays to the
device, run the library through its C ABI, and compare against the oracle."""
from __future__ import annotations

import numpy as np

import workloads as wl

TOL_FROB = 2e-3          # relative Frobenius error on C
TOL_REL, TOL_ABS = 1e-2, 1e-2  # elementwise |C - ref| <= TOL_REL |ref| + TOL_ABS


def torch_dtype(dt):
    import torch
    return torch.float16 if dt == wl.F16 else torch.bfloat16


def to_device(bits: np.ndarray | None, dt, offset_elems: int = 0):
    """uint16 bits -> CUDA tensor of the 16-bit float type.  With offset_elems > 0
    the tensor is a view that starts that many elements into a larger buffer
    (a base that is 2-byte but not 16-byte aligned)."""
    import torch
    if bits is None:
        return None
    flat = torch.from_numpy(np.ascontiguousarray(bits).reshape(-1).view(np.int16))
    if offset_elems:
        buf = torch.empty(flat.numel() + offset_elems, dtype=torch.int16)
        buf[offset_elems:] = flat
        dev = buf.cuda()[offset_elems:]
    else:
        dev = flat.cuda()
    return dev.view(torch_dtype(dt)).view(bits.shape)


def from_device(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def run_library(A_bits, B_bits, bias_bits, dt, epi, config=0, offsets=(0, 0, 0, 0), sync=True,
                b_transposed=False, out_f32=False, force_split=False):
    """C bits from tl_gemm (through the C ABI) for host bit arrays.  B_bits is
    K x N; with b_transposed the library is given its transpose (N x K).  With
    out_f32 the library writes float32 C and that float32 array is returned."""
    import torch
    import tensor_core_gemm_tl_b200 as tg
    A = to_device(A_bits, dt, offsets[0])
    B = to_device(np.ascontiguousarray(B_bits.T) if b_transposed else B_bits, dt, offsets[1])
    bias = to_device(bias_bits, dt, offsets[2]) if bias_bits is not None else None
    M, N = A_bits.shape[0], B_bits.shape[1]
    cdt = torch.float32 if out_f32 else torch_dtype(dt)
    if offsets[3]:
        buf = torch.empty(M * N + offsets[3], dtype=cdt, device="cuda")
        out = buf[offsets[3]:].view(M, N)
    else:
        out = torch.empty((M, N), dtype=cdt, device="cuda")
    tg.gemm(A, B, bias, epilogue=int(epi), out=out, config=config, b_transposed=b_transposed,
            force_split=force_split)
    if sync:
        torch.cuda.synchronize()
        assert tg.check_device() == 0
    return out.cpu().numpy() if out_f32 else from_device(out)


def round_to_dtype(x: np.ndarray, dt) -> np.ndarray:
    """fp64 -> the nearest fp16 / bf16 value (ties to even), returned as float64.
    Rounds once, directly from fp64 (no float32 step)."""
    p, qmin = (11, -24) if dt == wl.F16 else (8, -133)
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.exp2(np.maximum(e - p, qmin).astype(np.float64))
    return np.rint(x / q) * q


F32 = "f32"  # output-type tag for ulp() and accumulation_bound()


def ulp(v: np.ndarray, dt) -> np.ndarray:
    """Spacing of the fp16 / bf16 (or, for dt == F32, float32) values at
    magnitude |v| (subnormal spacing near 0)."""
    p, qmin = {wl.F16: (11, -24), wl.BF16: (8, -133), F32: (24, -149)}[dt]
    _, e = np.frexp(np.abs(np.asarray(v, dtype=np.float64)))
    return np.exp2(np.maximum(e - p, qmin).astype(np.float64))


def accumulation_bound(A_bits, B_bits, bias_bits, dt, epi, ref, rows=None, points=None, out_f32=False):
    """Worst-case |C - ref| of a correct kernel: an fp32 sum of K exact products
    (each addition rounded, or truncated, to fp32: relative error <= 2^-23 per
    step, so at most K 2^-23 sum_k |a_ik b_kj|), then for the epilogue the bias
    add and GELU in fp32 (|GELU'| <= 1.13 for both forms; the float32 erf GELU
    is within 1e-5 relative, the tanh form within 2e-5 down to x = -10 and
    its tail below that is covered by the absolute terms), then one rounding
    to the output type (half an ulp; float32 with out_f32)."""
    Af = wl.bits_to_float32(A_bits, dt).astype(np.float64)
    Bf = wl.bits_to_float32(B_bits, dt).astype(np.float64)
    K = Af.shape[1]
    if points is not None:
        ii, jj = points
        absdot = np.einsum("pk,kp->p", np.abs(Af[ii]), np.abs(Bf[:, jj]))
    else:
        Ar = Af if rows is None else Af[rows]
        absdot = np.abs(Ar) @ np.abs(Bf)
    e = K * 2.0 ** -23 * absdot
    if epi != wl.EPI_NONE:
        if bias_bits is not None and epi in wl.EPI_WITH_BIAS:
            b = np.abs(wl.bits_to_float32(bias_bits, dt).astype(np.float64))
            b = b[points[1]] if points is not None else b[None, :]
        else:
            b = 0.0
        rel = 2e-5 if epi in (wl.EPI_BIAS_GELU_TANH, wl.EPI_GELU_TANH) else 1e-5
        e = 1.2 * (e + 2.0 ** -22 * (absdot + b)) + rel * np.abs(ref)
    return 0.5 * ulp(np.abs(ref) + e, F32 if out_f32 else dt) + e + 1e-45


def ordered(bits: np.ndarray) -> np.ndarray:
    """Sign-magnitude 16-bit patterns -> integers whose difference counts ulps."""
    b = bits.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def compare(C_bits, ref, dt, bound=None):
    """Errors of the library's C against the oracle's fp64 reference; asserts
    the two stated tolerances and, when `bound` (elementwise, from
    accumulation_bound) is given, that every element lies within it."""
    C = wl.bits_to_float32(C_bits, dt).astype(np.float64)
    assert C.shape == ref.shape
    assert np.all(np.isfinite(C)), "non-finite output"
    diff = C - ref
    frob = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    viol = np.abs(diff) - (TOL_REL * np.abs(ref) + TOL_ABS)
    rn = wl.round_to_bits(round_to_dtype(ref, dt).astype(np.float32), dt)
    ulps = np.abs(ordered(C_bits) - ordered(rn))
    stats = {"rel_frobenius": frob, "max_abs_err": float(np.abs(diff).max()),
             "max_violation": float(viol.max()), "max_ulps_vs_rounded_ref": int(ulps.max())}
    assert frob <= TOL_FROB, stats
    assert viol.max() <= 0, stats
    if bound is not None:
        over = np.abs(diff) - bound
        stats["max_over_bound"] = float(over.max())
        assert over.max() <= 0, stats
    return stats


def compare_f32(C, ref, bound):
    """float32 C against the oracle's fp64 reference: the two stated
    tolerances and the elementwise bound (from accumulation_bound with
    out_f32=True)."""
    C = np.asarray(C, dtype=np.float64)
    assert C.shape == ref.shape
    assert np.all(np.isfinite(C)), "non-finite output"
    diff = C - ref
    frob = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    viol = np.abs(diff) - (TOL_REL * np.abs(ref) + TOL_ABS)
    over = np.abs(diff) - bound
    stats = {"rel_frobenius": frob, "max_abs_err": float(np.abs(diff).max()),
             "max_violation": float(viol.max()), "max_over_bound": float(over.max())}
    assert frob <= TOL_FROB, stats
    assert viol.max() <= 0, stats
    assert over.max() <= 0, stats
    return stats
