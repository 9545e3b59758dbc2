"""Pins for the oracle's attention forward: each checks it against something
other than the oracle (closed forms, mpmath, scipy's softmax, invariances).
Collected by test_oracle_pins.py; test_oracle_mutants.py plants mistakes."""
from __future__ import annotations

import math

import numpy as np

import workloads as wl

F16, BF16 = wl.F16, wl.BF16


def _bits(rng, shape, dt, scale=1.0):
    return wl.round_to_bits((rng.normal(size=shape) * scale).astype(np.float32), dt)


def _f64(bits, dt):
    return wl.bits_to_float32(bits, dt).astype(np.float64)


def pin_attn_uniform_when_q_is_zero(orc):
    """Q = 0: every kept key has weight 1/n, so O is the mean of the kept V rows
    and lse = log n (non-causal: n = Sk; causal: n = i + 1)."""
    rng = np.random.default_rng(31)
    for dt, causal in ((F16, False), (BF16, True), (F16, True)):
        B, H, Sq, Sk, D = 2, 3, 9, 9, 16
        Q = np.zeros((B, H, Sq, D), np.uint16)
        K = _bits(rng, (B, H, Sk, D), dt)
        V = _bits(rng, (B, H, Sk, D), dt)
        O, lse = orc.attention(Q, K, V, dt, causal, 0.25)
        Vf = _f64(V, dt)
        for i in range(Sq):
            n = i + 1 if causal else Sk
            mean = np.array([[[math.fsum(Vf[b, h, :n, d]) / n for d in range(D)] for h in range(H)]
                             for b in range(B)])
            assert np.allclose(O[:, :, i, :], mean, rtol=1e-13, atol=1e-15)
            assert np.allclose(lse[:, :, i], math.log(n), rtol=1e-14)


def pin_attn_vs_scipy_softmax(orc):
    """Random small shapes: scipy's softmax of the fp64 scores, times V."""
    from scipy.special import logsumexp, softmax
    rng = np.random.default_rng(37)
    for dt, causal, (Sq, Sk, D) in ((BF16, False, (7, 11, 8)), (F16, True, (12, 12, 16)),
                                    (BF16, True, (5, 9, 32)), (F16, False, (1, 1, 8))):
        Q = _bits(rng, (1, 2, Sq, D), dt)
        K = _bits(rng, (1, 2, Sk, D), dt)
        V = _bits(rng, (1, 2, Sk, D), dt)
        scale = 1 / math.sqrt(D)
        O, lse = orc.attention(Q, K, V, dt, causal, scale)
        S = np.einsum("bhqd,bhkd->bhqk", _f64(Q, dt), _f64(K, dt)) * scale
        if causal:
            S = np.where(np.arange(Sk)[None, :] <= np.arange(Sq)[:, None], S, -np.inf)
        ref = np.einsum("bhqk,bhkd->bhqd", softmax(S, axis=-1), _f64(V, dt))
        assert np.allclose(O, ref, rtol=1e-12, atol=1e-14)
        assert np.allclose(lse, logsumexp(S, axis=-1), rtol=1e-13, atol=1e-14)


def pin_attn_mpmath_tiny(orc):
    """Two queries over three keys, recomputed with mpmath at 40 digits."""
    import mpmath as mp
    mp.mp.dps = 40
    rng = np.random.default_rng(41)
    dt = BF16
    Q = _bits(rng, (1, 1, 2, 4), dt, 2.0)
    K = _bits(rng, (1, 1, 3, 4), dt, 2.0)
    V = _bits(rng, (1, 1, 3, 4), dt)
    O, lse = orc.attention(Q, K, V, dt, False, 0.7)
    q, k, v = _f64(Q, dt)[0, 0], _f64(K, dt)[0, 0], _f64(V, dt)[0, 0]
    for i in range(2):
        s = [mp.mpf(0.7) * mp.fsum(mp.mpf(q[i, d]) * mp.mpf(k[j, d]) for d in range(4)) for j in range(3)]
        w = [mp.e ** x for x in s]
        tot = mp.fsum(w)
        for d in range(4):
            ref = mp.fsum(w[j] * mp.mpf(v[j, d]) for j in range(3)) / tot
            assert abs(O[0, 0, i, d] - float(ref)) <= 1e-14 * (abs(float(ref)) + 1e-3)
        assert abs(lse[0, 0, i] - float(mp.log(tot))) <= 1e-14 * abs(float(mp.log(tot))) + 1e-15


def pin_attn_single_key_and_first_causal_row(orc):
    """One key: the weight is 1, O = V[0] exactly and lse = scale q.k.  Causal:
    query 0 sees only key 0, so O[0] = V[0] exactly."""
    rng = np.random.default_rng(43)
    for dt in (F16, BF16):
        Q = _bits(rng, (2, 2, 4, 8), dt)
        K = _bits(rng, (2, 2, 1, 8), dt)
        V = _bits(rng, (2, 2, 1, 8), dt)
        O, lse = orc.attention(Q, K, V, dt, False, 0.5)
        assert np.array_equal(O, np.broadcast_to(_f64(V, dt), O.shape))
        qk = np.einsum("bhqd,bhkd->bhq", _f64(Q, dt), _f64(K, dt)) * 0.5
        assert np.allclose(lse, qk, rtol=1e-15, atol=1e-15)
        K2 = _bits(rng, (2, 2, 6, 8), dt)
        V2 = _bits(rng, (2, 2, 6, 8), dt)
        O2, _ = orc.attention(_bits(rng, (2, 2, 6, 8), dt), K2, V2, dt, True, 0.5)
        assert np.array_equal(O2[:, :, 0, :], _f64(V2, dt)[:, :, 0, :])


def pin_attn_hard_attention(orc):
    """Scores far apart: the largest takes all the weight (exp(-2000) is 0 in
    fp64), so O is that key's V row exactly; without subtracting the maximum
    the exponentials would overflow."""
    dt = F16
    D, Sk = 8, 5
    Q = wl.round_to_bits(np.eye(1, D, dtype=np.float32).reshape(1, 1, 1, D) * 64, dt)
    kvals = np.array([10.0, 40.0, 20.0, -30.0, 5.0], np.float32)
    Kf = np.zeros((1, 1, Sk, D), np.float32)
    Kf[0, 0, :, 0] = kvals
    K = wl.round_to_bits(Kf, dt)
    V = _bits(np.random.default_rng(47), (1, 1, Sk, D), dt)
    O, lse = orc.attention(Q, K, V, dt, False, 1.0)
    assert np.array_equal(O[0, 0, 0], _f64(V, dt)[0, 0, 1])
    assert lse[0, 0, 0] == 64.0 * 40.0


def pin_attn_key_permutation(orc):
    """Non-causal attention does not depend on the order of the keys (K and V
    permuted together), up to fp64 summation order."""
    rng = np.random.default_rng(53)
    dt = BF16
    Q = _bits(rng, (1, 2, 6, 16), dt)
    K = _bits(rng, (1, 2, 10, 16), dt)
    V = _bits(rng, (1, 2, 10, 16), dt)
    perm = rng.permutation(10)
    O1, l1 = orc.attention(Q, K, V, dt, False, 0.3)
    O2, l2 = orc.attention(Q, np.ascontiguousarray(K[:, :, perm]), np.ascontiguousarray(V[:, :, perm]),
                           dt, False, 0.3)
    assert np.allclose(O1, O2, rtol=1e-13, atol=1e-15) and np.allclose(l1, l2, rtol=1e-14)


def pin_attn_rows_match_full(orc):
    rng = np.random.default_rng(59)
    dt = F16
    Q = _bits(rng, (2, 2, 7, 8), dt)
    K = _bits(rng, (2, 2, 9, 8), dt)
    V = _bits(rng, (2, 2, 9, 8), dt)
    O, lse = orc.attention(Q, K, V, dt, True, 0.4)
    bh = np.array([3, 0, 2, 1])
    qi = np.array([6, 0, 3, 5])
    Or, lr = orc.attention(Q, K, V, dt, True, 0.4, rows=(bh, qi))
    assert np.array_equal(Or, O.reshape(4, 7, 8)[bh, qi]) and np.array_equal(lr, lse.reshape(4, 7)[bh, qi])


ATTENTION_PINS = [
    pin_attn_uniform_when_q_is_zero, pin_attn_vs_scipy_softmax, pin_attn_mpmath_tiny,
    pin_attn_single_key_and_first_causal_row, pin_attn_hard_attention, pin_attn_key_permutation,
    pin_attn_rows_match_full,
]
