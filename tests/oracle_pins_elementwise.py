"""Pins for the oracle's row softmax and vector add."""
from __future__ import annotations

import numpy as np

import workloads as wl


def pin_softmax_closed_forms(orc):
    """A constant row gives 1/n everywhere; a row with one entry far above the
    rest gives the indicator of that entry (the others underflow to 0)."""
    for dt in (wl.F16, wl.BF16):
        X = wl.round_to_bits(np.full((3, 37), 2.5, np.float32), dt)
        assert np.array_equal(orc.softmax_rows(X, dt), np.full((3, 37), 1.0 / 37))
        x = np.full((1, 9), -30000.0 if dt == wl.F16 else -1e30, np.float32)
        x[0, 4] = 0.0
        Y = orc.softmax_rows(wl.round_to_bits(x, dt), dt)
        assert np.array_equal(Y[0], np.eye(1, 9, 4)[0])


def pin_softmax_vs_scipy(orc):
    from scipy.special import softmax
    rng = np.random.default_rng(61)
    for dt, (r, c) in ((wl.F16, (5, 1000)), (wl.BF16, (7, 33)), (wl.BF16, (1, 1))):
        X = wl.round_to_bits((rng.normal(size=(r, c)) * 4).astype(np.float32), dt)
        ref = softmax(wl.bits_to_float32(X, dt).astype(np.float64), axis=1)
        assert np.allclose(orc.softmax_rows(X, dt), ref, rtol=1e-13, atol=1e-300)


def pin_softmax_shift_invariance(orc):
    """Adding a constant to a row (exact in bf16 at these values) leaves the
    softmax unchanged up to fp64 rounding, and each row sums to one."""
    rng = np.random.default_rng(67)
    dt = wl.BF16
    x = np.round(rng.normal(size=(4, 50)) * 8).astype(np.float32)  # small integers: shifts stay exact
    Y1 = orc.softmax_rows(wl.round_to_bits(x, dt), dt)
    Y2 = orc.softmax_rows(wl.round_to_bits(x + 64.0, dt), dt)
    assert np.allclose(Y1, Y2, rtol=1e-14, atol=1e-300)
    assert np.allclose(Y1.sum(axis=1), 1.0, rtol=1e-14)


def pin_vector_add(orc):
    """Bit for bit numpy's float32 addition; commutative; x + 0 = x."""
    rng = np.random.default_rng(71)
    A = (rng.normal(size=10007) * 1e3).astype(np.float32)
    B = (rng.normal(size=10007) * 1e-3).astype(np.float32)
    assert np.array_equal(orc.vector_add(A, B), A + B)
    assert np.array_equal(orc.vector_add(A, B), orc.vector_add(B, A))
    assert np.array_equal(orc.vector_add(A, np.zeros_like(A)), A)


ELEMENTWISE_PINS = [pin_softmax_closed_forms, pin_softmax_vs_scipy, pin_softmax_shift_invariance, pin_vector_add]
