"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when that oracle disagrees with an independent source of truth:

  * exact rational arithmetic (Python ``fractions.Fraction``) on tiny shapes,
  * closed forms (identity, all-ones, row sums, B = 0),
  * the standard normal table (textbook Phi values, tests/golden),
  * library routines (numpy fp64 matmul, numpy / torch float decoding,
    scipy's normal CDF, mpmath's high-precision erf),
  * invariants (transpose, power-of-two scaling, GELU odd-part identity).

They are collected by test_oracle_pins.py, and test_oracle_mutants.py runs
them against copies of the oracle with a planted mistake to show that each
plausible mistake fails at least one pin.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

import workloads as wl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
F16, BF16 = wl.F16, wl.BF16
EPI_NONE, EPI_BIAS_GELU = wl.EPI_NONE, wl.EPI_BIAS_GELU
U53 = 2.0 ** -53


def load_phi_table():
    xs, ps = [], []
    with open(os.path.join(GOLDEN, "normal_cdf_table.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            x, p = line.split()
            xs.append(float(x))
            ps.append(float(p))
    return np.array(xs), np.array(ps)


def load_hand_example():
    mats, cur, rows = {}, None, 0
    with open(os.path.join(GOLDEN, "matmul_hand_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            if tok[0] in ("A", "B", "C"):
                cur, rows = tok[0], int(tok[1])
                mats[cur] = []
            else:
                mats[cur].append([float(t) for t in tok])
    return {k: np.array(v) for k, v in mats.items()}


def rand_bits(rng, shape, dtype, scale=1.0, kind="uniform"):
    if kind == "uniform":
        x = rng.uniform(-scale, scale, size=shape)
    else:
        x = rng.normal(0.0, scale, size=shape)
    return wl.round_to_bits(x.astype(np.float32), dtype)


def exact_values(bits, dtype):
    """Fractions equal to the fp16 / bf16 values (via float32, which holds both exactly)."""
    f32 = wl.bits_to_float32(bits, dtype)
    return [[Fraction(float(v)) for v in row] for row in np.atleast_2d(f32)]


# ---------------------------------------------------------------- decoding
def pin_decode_all_patterns(orc):
    """Every one of the 2^16 patterns decodes like numpy's float16 and like bf16's
    definition as the upper half of a float32 (torch agrees, checked elsewhere)."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref16 = allbits.view(np.float16).astype(np.float64)
    got16 = orc.decode(allbits, F16)
    assert np.array_equal(np.isnan(ref16), np.isnan(got16))
    ok = ~np.isnan(ref16)
    assert np.array_equal(ref16[ok], got16[ok]), "fp16 decode"
    assert np.array_equal(np.signbit(ref16[ok]), np.signbit(got16[ok])), "fp16 signed zero"
    with np.errstate(invalid="ignore"):
        refbf = (allbits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    gotbf = orc.decode(allbits, BF16)
    assert np.array_equal(np.isnan(refbf), np.isnan(gotbf))
    ok = ~np.isnan(refbf)
    assert np.array_equal(refbf[ok], gotbf[ok]), "bf16 decode"


# ---------------------------------------------------------------- GEMM part
def pin_hand_example(orc):
    g = load_hand_example()
    for dt in (F16, BF16):
        A = wl.round_to_bits(g["A"].astype(np.float32), dt)
        B = wl.round_to_bits(g["B"].astype(np.float32), dt)
        C = orc.gemm(A, B, None, dt, EPI_NONE)
        assert np.array_equal(C, g["C"]), (dt, C)


def pin_exact_bruteforce(orc, cases=40, seed=1234):
    """Shapes up to 8x8x8: the oracle equals the exact rational product rounded
    to fp64, within the fp64 summation bound (K-1) u sum|a b|."""
    rng = np.random.default_rng(seed)
    for t in range(cases):
        dt = (F16, BF16)[t % 2]
        M, N, K = (int(v) for v in rng.integers(1, 9, size=3))
        kind = ("uniform", "normal")[(t // 2) % 2]
        A = rand_bits(rng, (M, K), dt, 1.0, kind)
        B = rand_bits(rng, (K, N), dt, 4.0, kind)
        C = orc.gemm(A, B, None, dt, EPI_NONE)
        Ae, Be = exact_values(A, dt), exact_values(B, dt)
        for i in range(M):
            for j in range(N):
                exact = sum((Ae[i][k] * Be[k][j] for k in range(K)), Fraction(0))
                mag = float(sum((abs(Ae[i][k] * Be[k][j]) for k in range(K)), Fraction(0)))
                err = abs(Fraction(C[i, j]) - exact)
                assert float(err) <= max(K - 1, 0) * U53 * mag + 1e-300, (t, i, j, float(err))


def pin_exact_bruteforce_epilogue(orc, cases=24, seed=99):
    """With bias+GELU: x = exact sum + bias, GELU(x) = x (1 + erf(x / sqrt 2)) / 2
    evaluated by mpmath at 40 digits."""
    import mpmath
    mpmath.mp.dps = 40
    rng = np.random.default_rng(seed)
    for t in range(cases):
        dt = (F16, BF16)[t % 2]
        M, N, K = (int(v) for v in rng.integers(1, 9, size=3))
        A = rand_bits(rng, (M, K), dt, 1.0)
        B = rand_bits(rng, (K, N), dt, 1.0)
        bias = rand_bits(rng, (N,), dt, 1.0, "normal")
        C = orc.gemm(A, B, bias, dt, EPI_BIAS_GELU)
        Ae, Be = exact_values(A, dt), exact_values(B, dt)
        be = exact_values(bias, dt)[0]
        for i in range(M):
            for j in range(N):
                x = sum((Ae[i][k] * Be[k][j] for k in range(K)), Fraction(0)) + be[j]
                xm = mpmath.mpf(x.numerator) / x.denominator
                ref = float(xm * (1 + mpmath.erf(xm / mpmath.sqrt(2))) / 2)
                assert abs(C[i, j] - ref) <= 1e-14 * (abs(ref) + abs(float(x))) + 1e-300, (t, i, j)


def pin_vs_numpy_matmul(orc, seed=7):
    """No epilogue: numpy's fp64 matmul of the decoded operands, to fp64 accuracy."""
    rng = np.random.default_rng(seed)
    for dt, (M, N, K) in ((F16, (37, 61, 53)), (BF16, (64, 23, 130)), (F16, (5, 300, 257))):
        A = rand_bits(rng, (M, K), dt, 1.0, "normal")
        B = rand_bits(rng, (K, N), dt, 1.0, "uniform")
        Af = wl.bits_to_float32(A, dt).astype(np.float64)
        Bf = wl.bits_to_float32(B, dt).astype(np.float64)
        ref = Af @ Bf
        bound = 2 * K * U53 * (np.abs(Af) @ np.abs(Bf))
        C = orc.gemm(A, B, None, dt, EPI_NONE)
        assert np.all(np.abs(C - ref) <= bound + 1e-300), (dt, M, N, K)


def pin_identity(orc, seed=3):
    """A = I (M = K)  =>  C = B exactly."""
    rng = np.random.default_rng(seed)
    for dt, (n, N) in ((F16, (24, 17)), (BF16, (40, 9))):
        A = wl.round_to_bits(np.eye(n, dtype=np.float32), dt)
        B = rand_bits(rng, (n, N), dt, 3.0, "normal")
        C = orc.gemm(A, B, None, dt, EPI_NONE)
        assert np.array_equal(C, wl.bits_to_float32(B, dt).astype(np.float64))
        # and the other side: B = I  =>  C = A
        A2 = rand_bits(rng, (N, n), dt, 3.0, "normal")
        B2 = wl.round_to_bits(np.eye(n, dtype=np.float32), dt)
        C2 = orc.gemm(A2, B2, None, dt, EPI_NONE)
        assert np.array_equal(C2, wl.bits_to_float32(A2, dt).astype(np.float64))


def pin_row_sums(orc, seed=5):
    """B = all ones  =>  C[i, j] = sum_k A[i, k] (exact here: the fp16 values are
    multiples of 2^-24 below 1 and K <= 32, so every partial sum is exact)."""
    rng = np.random.default_rng(seed)
    for dt, (M, N, K) in ((F16, (9, 5, 32)), (BF16, (7, 11, 19))):
        A = rand_bits(rng, (M, K), dt, 1.0)
        B = wl.round_to_bits(np.ones((K, N), np.float32), dt)
        C = orc.gemm(A, B, None, dt, EPI_NONE)
        Af = wl.bits_to_float32(A, dt).astype(np.float64)
        sums = np.array([math.fsum(r) for r in Af])
        assert np.array_equal(C, np.repeat(sums[:, None], N, axis=1))


def pin_all_ones(orc):
    """A = B = all ones  =>  C = K everywhere."""
    for dt in (F16, BF16):
        for K in (1, 7, 64, 2048, 4096):
            A = wl.round_to_bits(np.ones((3, K), np.float32), dt)
            B = wl.round_to_bits(np.ones((K, 4), np.float32), dt)
            assert np.all(orc.gemm(A, B, None, dt, EPI_NONE) == K)


def pin_zero_B_gelu_table(orc):
    """B = 0 with bias+GELU  =>  C[i, j] = GELU(bias[j]) = bias[j] * Phi(bias[j]),
    with Phi from the standard normal table: pins the bias-before-GELU order
    and the exact-GELU form independently of any erf routine."""
    xs, ps = load_phi_table()
    xs_all = np.concatenate([xs, -xs[1:]])
    phi_all = np.concatenate([ps, 1.0 - ps[1:]])
    for dt in (F16, BF16):
        bias = wl.round_to_bits(xs_all.astype(np.float32), dt)
        assert np.array_equal(wl.bits_to_float32(bias, dt), xs_all.astype(np.float32))
        K, M, N = 5, 3, xs_all.size
        A = wl.round_to_bits(np.ones((M, K), np.float32), dt)
        B = np.zeros((K, N), np.uint16)
        C = orc.gemm(A, B, bias, dt, EPI_BIAS_GELU)
        expect = xs_all * phi_all
        assert np.all(np.abs(C - expect[None, :]) <= 6e-11 * np.maximum(np.abs(xs_all), 1.0)), C


def pin_bias_then_gelu(orc, seed=11):
    """x = (A.B)[i, j] + bias[j], then x * Phi(x) with scipy's normal CDF."""
    from scipy.stats import norm
    rng = np.random.default_rng(seed)
    for dt, (M, N, K) in ((F16, (13, 29, 40)), (BF16, (8, 33, 64))):
        A = rand_bits(rng, (M, K), dt, 1.0)
        B = rand_bits(rng, (K, N), dt, 1.0 / math.sqrt(K), "normal")
        bias = rand_bits(rng, (N,), dt, 1.0, "normal")
        plain = orc.gemm(A, B, None, dt, EPI_NONE)
        fused = orc.gemm(A, B, bias, dt, EPI_BIAS_GELU)
        x = plain + wl.bits_to_float32(bias, dt).astype(np.float64)[None, :]
        ref = x * norm.cdf(x)
        assert np.all(np.abs(fused - ref) <= 1e-14 * (np.abs(x) + 1e-300) + 1e-300)


def pin_transpose(orc, seed=13):
    """(A B)^T = B^T A^T, bit for bit (same products, same k order)."""
    rng = np.random.default_rng(seed)
    for dt, (M, N, K) in ((F16, (19, 7, 33)), (BF16, (6, 21, 10))):
        A = rand_bits(rng, (M, K), dt, 1.0, "normal")
        B = rand_bits(rng, (K, N), dt, 1.0, "normal")
        C = orc.gemm(A, B, None, dt, EPI_NONE)
        Ct = orc.gemm(np.ascontiguousarray(B.T), np.ascontiguousarray(A.T), None, dt, EPI_NONE)
        assert np.array_equal(C.T, Ct)


def pin_power_of_two_scaling(orc, seed=17):
    """oracle(2^p A, B) = 2^p oracle(A, B) exactly (no epilogue)."""
    rng = np.random.default_rng(seed)
    for dt in (F16, BF16):
        A = rand_bits(rng, (11, 20), dt, 1.0)
        B = rand_bits(rng, (20, 9), dt, 1.0)
        for p in (-3, 1, 4):
            A2 = wl.round_to_bits(wl.bits_to_float32(A, dt) * np.float32(2.0 ** p), dt)
            assert np.array_equal(wl.bits_to_float32(A2, dt),
                                  wl.bits_to_float32(A, dt) * np.float32(2.0 ** p))
            assert np.array_equal(orc.gemm(A2, B, None, dt, EPI_NONE),
                                  orc.gemm(A, B, None, dt, EPI_NONE) * 2.0 ** p)


def pin_rows_and_points(orc, seed=19):
    """The row-subset and single-point entry points agree bit for bit with the
    whole product, in every epilogue mode."""
    rng = np.random.default_rng(seed)
    M, N, K = 23, 31, 45
    for dt in (F16, BF16):
        A = rand_bits(rng, (M, K), dt, 1.0)
        B = rand_bits(rng, (K, N), dt, 1.0)
        bias = rand_bits(rng, (N,), dt, 0.5, "normal")
        for epi, b in ((EPI_NONE, None), (EPI_BIAS_GELU, bias), (wl.EPI_BIAS, bias), (wl.EPI_GELU, None),
                       (wl.EPI_BIAS_GELU_TANH, bias), (wl.EPI_GELU_TANH, None)):
            full = orc.gemm(A, B, b, dt, epi)
            rows = np.array([22, 0, 5, 5, 17])
            assert np.array_equal(orc.gemm(A, B, b, dt, epi, rows=rows), full[rows])
            ii = rng.integers(0, M, 50)
            jj = rng.integers(0, N, 50)
            assert np.array_equal(orc.gemm_points(A, B, b, dt, epi, ii, jj), full[ii, jj])


def pin_bias_only_and_gelu_only(orc, seed=29):
    """Bias-only: numpy's fp64 matmul plus the bias row.  GELU-only with A = I:
    C = GELU(B) elementwise, checked on the standard normal table."""
    rng = np.random.default_rng(seed)
    for dt, (M, N, K) in ((F16, (9, 17, 33)), (BF16, (12, 8, 40))):
        A = rand_bits(rng, (M, K), dt, 1.0)
        B = rand_bits(rng, (K, N), dt, 1.0)
        bias = rand_bits(rng, (N,), dt, 1.0, "normal")
        Af = wl.bits_to_float32(A, dt).astype(np.float64)
        Bf = wl.bits_to_float32(B, dt).astype(np.float64)
        ref = Af @ Bf + wl.bits_to_float32(bias, dt).astype(np.float64)[None, :]
        got = orc.gemm(A, B, bias, dt, wl.EPI_BIAS)
        assert np.all(np.abs(got - ref) <= 2 * K * U53 * (np.abs(Af) @ np.abs(Bf) + 1) + 1e-300)
    xs, ps = load_phi_table()
    xs_all = np.concatenate([xs, -xs[1:]])
    phi_all = np.concatenate([ps, 1.0 - ps[1:]])
    for dt in (F16, BF16):
        n = xs_all.size
        A = wl.round_to_bits(np.eye(n, dtype=np.float32), dt)
        B = wl.round_to_bits(np.tile(xs_all.astype(np.float32), (n, 1)), dt)  # every row = the table
        got = orc.gemm(A, B, None, dt, wl.EPI_GELU)
        expect = (xs_all * phi_all)[None, :]
        assert np.all(np.abs(got - expect) <= 6e-11 * np.maximum(np.abs(xs_all), 1.0)[None, :])


# ---------------------------------------------------------------- GELU alone
def pin_gelu_table(orc):
    xs, ps = load_phi_table()
    for x, p in zip(xs, ps):
        for s in (1.0, -1.0):
            xv = s * x
            ref = xv * (p if s > 0 else 1.0 - p)
            got = orc.gelu(np.array([xv]))[0]
            assert abs(got - ref) <= 6e-11 * max(abs(xv), 1.0), (xv, got, ref)


def pin_gelu_invariants(orc, seed=23):
    rng = np.random.default_rng(seed)
    assert orc.gelu(np.array([0.0]))[0] == 0.0
    x = rng.normal(0, 3, 1000)
    # GELU(x) - GELU(-x) = x (Phi(x) + Phi(-x)) = x
    d = orc.gelu(x) - orc.gelu(-x)
    assert np.all(np.abs(d - x) <= 1e-15 * (np.abs(x) + 1)), "odd part"
    big = np.linspace(6, 60, 50)
    assert np.all(np.abs(orc.gelu(big) - big) < 1e-8 * big)
    assert np.all(orc.gelu(-big) <= 0) and np.all(orc.gelu(-big) > -1e-8)
    # increasing for x >= 0
    xs = np.linspace(0, 10, 2001)
    assert np.all(np.diff(orc.gelu(xs)) > 0)


def pin_gelu_tail_relative(orc):
    """Relative accuracy of GELU over the whole range, the far negative tail
    included (where x * Phi(x) is tiny): mpmath at 40 digits."""
    import mpmath
    mpmath.mp.dps = 40
    xs = np.concatenate([np.linspace(-35, -1, 300), np.linspace(1, 30, 100), [-0.3, 0.25]])
    got = orc.gelu(xs)
    for x, g in zip(xs, got):
        ref = float(mpmath.mpf(x) * mpmath.ncdf(mpmath.mpf(x)))
        # the rounding of x / sqrt 2 alone moves erfc by ~2 z^2 u relative (z = |x| / sqrt 2)
        assert abs(g - ref) <= (1e-15 + 4e-16 * x * x) * abs(ref), (x, g, ref)


# ---------------------------------------------------------------- tanh-form GELU
def _mp_gelu_tanh(x):
    """0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), the GELU paper's tanh
    approximation, in mpmath (the caller sets the precision)."""
    import mpmath
    # 1 + tanh(u) loses about 0.87 |u| digits for u << 0: carry that many more
    u = abs(0.7978845608028654 * (x + 0.044715 * x ** 3))
    with mpmath.workdps(mpmath.mp.dps + int(0.87 * u) + 10):
        xm = mpmath.mpf(x)
        return +(xm / 2 * (1 + mpmath.tanh(mpmath.sqrt(2 / mpmath.pi) * (xm + mpmath.mpf("0.044715") * xm ** 3))))


def pin_gelu_tanh_mpmath(orc):
    """Relative accuracy over [-30, 30], tails included: mpmath at 40 digits."""
    import mpmath
    mpmath.mp.dps = 40
    xs = np.concatenate([np.linspace(-30, -1, 300), np.linspace(-1, 1, 41), np.linspace(1, 30, 100)])
    got = orc.gelu_tanh(xs)
    for x, g in zip(xs, got):
        ref = float(_mp_gelu_tanh(x))
        # exp(-2u) carries the rounding of u: about |2u| u53 relative
        u2 = abs(2 * 0.7978845608028654 * (x + 0.044715 * x ** 3))
        assert abs(g - ref) <= (2e-15 + 4e-16 * u2) * abs(ref) + 1e-320, (x, g, ref)


def pin_gelu_tanh_invariants(orc, seed=37):
    """g(0) = 0; g(x) - g(-x) = x; and the approximation stays within its known
    distance of the erf form (largest gap 4.7e-4, near x = -2.7)."""
    rng = np.random.default_rng(seed)
    assert orc.gelu_tanh(np.array([0.0]))[0] == 0.0
    x = rng.normal(0, 3, 1000)
    d = orc.gelu_tanh(x) - orc.gelu_tanh(-x)
    assert np.all(np.abs(d - x) <= 1e-15 * (np.abs(x) + 1)), "odd part"
    xs = np.linspace(-8, 8, 3201)
    gap = np.max(np.abs(orc.gelu_tanh(xs) - orc.gelu(xs)))
    assert 4.5e-4 < gap < 5.0e-4, gap


def pin_exact_bruteforce_tanh_epilogue(orc, cases=16, seed=101):
    """Bias + tanh GELU on tiny shapes: exact sum + bias (Fractions), then the
    tanh form in mpmath; and tanh GELU alone with A = I: C = g(B)."""
    import mpmath
    mpmath.mp.dps = 40
    rng = np.random.default_rng(seed)
    for t in range(cases):
        dt = (F16, BF16)[t % 2]
        M, N, K = (int(v) for v in rng.integers(1, 9, size=3))
        A = rand_bits(rng, (M, K), dt, 1.0)
        B = rand_bits(rng, (K, N), dt, 1.0)
        bias = rand_bits(rng, (N,), dt, 1.0, "normal")
        C = orc.gemm(A, B, bias, dt, wl.EPI_BIAS_GELU_TANH)
        Ae, Be = exact_values(A, dt), exact_values(B, dt)
        be = exact_values(bias, dt)[0]
        for i in range(M):
            for j in range(N):
                x = sum((Ae[i][k] * Be[k][j] for k in range(K)), Fraction(0)) + be[j]
                ref = float(_mp_gelu_tanh(mpmath.mpf(x.numerator) / x.denominator))
                assert abs(C[i, j] - ref) <= 1e-14 * (abs(ref) + abs(float(x))) + 1e-300, (t, i, j)
    for dt in (F16, BF16):
        n = 12
        A = wl.round_to_bits(np.eye(n, dtype=np.float32), dt)
        B = rand_bits(rng, (n, n), dt, 4.0, "normal")
        C = orc.gemm(A, B, None, dt, wl.EPI_GELU_TANH)
        Bf = wl.bits_to_float32(B, dt)
        for i in range(n):
            for j in range(n):
                ref = float(_mp_gelu_tanh(float(Bf[i, j])))
                assert abs(C[i, j] - ref) <= 1e-14 * (abs(ref) + 1e-3), (i, j)


ALL_PINS = [
    pin_decode_all_patterns, pin_hand_example, pin_exact_bruteforce,
    pin_exact_bruteforce_epilogue, pin_vs_numpy_matmul, pin_identity, pin_row_sums,
    pin_all_ones, pin_zero_B_gelu_table, pin_bias_then_gelu, pin_transpose,
    pin_power_of_two_scaling, pin_rows_and_points, pin_gelu_table, pin_gelu_invariants,
    pin_gelu_tail_relative, pin_bias_only_and_gelu_only,
    pin_gelu_tanh_mpmath, pin_gelu_tanh_invariants, pin_exact_bruteforce_tanh_epilogue,
]
