"""Attention forward on the GPU (through the C ABI) against the fp64 oracle.

Bar: every element of O within the error of a correct FlashAttention-style
kernel -- the softmax weights are rounded to the 16-bit input type before the
product with V (relative error 2^-9 for bf16, 2^-12 for fp16), so
|O - ref| <= 2 u (sum_j w_j |v_j| + |ref|) + half an output ulp -- and the
relative Frobenius error of O at most 1e-2; lse within 1e-4 (1 + |lse|)."""
import math
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
import workloads as wl  # noqa: E402
from gpu_util import from_device, to_device, ulp  # noqa: E402

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def make_qkv(B, H, Sq, Sk, D, dt, seed, q_scale=1.0):
    rng = np.random.default_rng(seed)
    Q = wl.round_to_bits((rng.normal(size=(B, H, Sq, D)) * q_scale).astype(np.float32), dt)
    K = wl.round_to_bits(rng.normal(size=(B, H, Sk, D)).astype(np.float32), dt)
    V = wl.round_to_bits(rng.normal(size=(B, H, Sk, D)).astype(np.float32), dt)
    return Q, K, V


def run_attention(Q, K, V, dt, causal, scale):
    import tensor_core_gemm_tl_b200 as tg
    q, k, v = to_device(Q, dt), to_device(K, dt), to_device(V, dt)
    B, H, Sq, D = Q.shape
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device="cuda")
    out = tg.attention(q, k, v, causal=causal, scale=scale, lse=lse)
    torch.cuda.synchronize()
    assert tg.check_device() == 0
    return from_device(out), lse.cpu().numpy().astype(np.float64)


def weighted_abs(Q, K, V, dt, causal, scale):
    """sum_j w_j |v_j| per output element, from fp64 softmax weights (test side)."""
    q = wl.bits_to_float32(Q, dt).astype(np.float64)
    k = wl.bits_to_float32(K, dt).astype(np.float64)
    v = np.abs(wl.bits_to_float32(V, dt).astype(np.float64))
    S = np.einsum("bhqd,bhkd->bhqk", q, k) * scale
    Sq, Sk = S.shape[2], S.shape[3]
    if causal:
        S = np.where(np.arange(Sk)[None, :] <= np.arange(Sq)[:, None], S, -np.inf)
    S = S - S.max(axis=-1, keepdims=True)
    W = np.exp(S)
    W /= W.sum(axis=-1, keepdims=True)
    return np.einsum("bhqk,bhkd->bhqd", W, v)


def check(O_bits, lse, Q, K, V, dt, causal, scale):
    ref, ref_lse = oracle.attention(Q, K, V, dt, causal, scale)
    got = wl.bits_to_float32(O_bits, dt).astype(np.float64)
    assert np.all(np.isfinite(got))
    u = 2.0 ** -9 if dt == wl.BF16 else 2.0 ** -12
    bound = 2 * u * (weighted_abs(Q, K, V, dt, causal, scale) + np.abs(ref)) + 0.5 * ulp(np.abs(ref), dt) + 1e-7
    err = np.abs(got - ref)
    frob = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert frob <= 1e-2, frob
    assert np.all(err <= bound), (err.max(), (err - bound).max())
    assert np.all(np.abs(lse - ref_lse) <= 1e-4 * (1 + np.abs(ref_lse))), np.abs(lse - ref_lse).max()
    return frob


CASES = [
    # B, H, Sq, Sk, D
    (1, 1, 128, 128, 64),
    (2, 3, 200, 333, 64),
    (1, 2, 256, 256, 128),
    (2, 2, 129, 57, 128),
    (1, 1, 1, 1, 64),
    (1, 2, 300, 500, 128),
    (1, 4, 512, 512, 64),
    # head_dim 128 past 256 queries runs on CTA pairs (512 query rows per pair):
    # ragged query counts, fewer and more keys than queries, several pairs
    (1, 2, 1000, 777, 128),
    (2, 1, 513, 1030, 128),
    (1, 1, 1536, 1536, 128),
]


@pytest.mark.parametrize("B,H,Sq,Sk,D", CASES)
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
@pytest.mark.parametrize("causal", [False, True])
def test_attention_vs_oracle(B, H, Sq, Sk, D, dt, causal):
    Q, K, V = make_qkv(B, H, Sq, Sk, D, dt, seed=Sq + Sk + D)
    scale = 1.0 / math.sqrt(D)
    O, lse = run_attention(Q, K, V, dt, causal, scale)
    check(O, lse, Q, K, V, dt, causal, scale)


def test_attention_long_sequence_rescaling():
    """Many key blocks and a growing running maximum: 4096 keys, scores
    scaled up so the maximum moves often."""
    dt, D = wl.BF16, 128
    Q, K, V = make_qkv(1, 2, 256, 4096, D, dt, seed=3, q_scale=3.0)
    for causal in (False, True):
        O, lse = run_attention(Q, K, V, dt, causal, 0.2)
        check(O, lse, Q, K, V, dt, causal, 0.2)


def test_attention_uniform_weights_give_the_mean_of_v():
    dt, D = wl.F16, 64
    Q = np.zeros((1, 1, 128, D), np.uint16)
    _, K, V = make_qkv(1, 1, 128, 384, D, dt, seed=5)
    O, lse = run_attention(Q, K, V, dt, False, 0.125)
    mean = wl.bits_to_float32(V, dt).astype(np.float64).mean(axis=2)
    got = wl.bits_to_float32(O, dt).astype(np.float64)
    assert np.all(np.abs(got - mean[:, :, None, :]) <= ulp(np.abs(mean[:, :, None, :]), dt) + 1e-6)
    assert np.allclose(lse, math.log(384), atol=1e-5)


def test_attention_deterministic():
    dt = wl.BF16
    Q, K, V = make_qkv(2, 2, 300, 700, 128, dt, seed=9)
    a, la = run_attention(Q, K, V, dt, True, 0.1)
    b, lb = run_attention(Q, K, V, dt, True, 0.1)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_attention_deterministic_with_every_sm_busy(causal, D):
    """Full-size launches (every SM holds a CTA for many rounds), repeated:
    the outputs agree bit for bit, so no ordering between a tile's P V and
    its next S (which overwrites the P that P V reads) varies from run to run."""
    dt = wl.BF16
    B, H, S = (4, 16, 4096) if D == 128 else (8, 16, 2048)
    Q, K, V = make_qkv(B, H, S, S, D, dt, seed=21)
    first, first_lse = run_attention(Q, K, V, dt, causal, 1.0 / math.sqrt(D))
    for _ in range(3):
        again, again_lse = run_attention(Q, K, V, dt, causal, 1.0 / math.sqrt(D))
        assert np.array_equal(first, again) and np.array_equal(first_lse, again_lse)


def weighted_abs_rows(Q, K, V, dt, causal, scale, bh, qi):
    """sum_j w_j |v_j| for the listed (batch*head, query) rows only, one row
    at a time (a head's K and V are read per row, not gathered for all)."""
    B, H, Sq, D = Q.shape
    Sk = K.shape[2]
    Qr, Kr, Vr = Q.reshape(B * H, Sq, D), K.reshape(B * H, Sk, D), V.reshape(B * H, Sk, D)
    out = np.empty((bh.size, D))
    for n, (h, i) in enumerate(zip(bh, qi)):
        q = wl.bits_to_float32(Qr[h, i], dt).astype(np.float64)
        k = wl.bits_to_float32(Kr[h], dt).astype(np.float64)
        v = np.abs(wl.bits_to_float32(Vr[h], dt).astype(np.float64))
        s = k @ q * scale
        if causal:
            s[i + 1:] = -np.inf
        w = np.exp(s - s.max())
        out[n] = (w / w.sum()) @ v
    return out


@pytest.mark.parametrize("dt", [wl.BF16, wl.F16])
@pytest.mark.parametrize("causal", [False, True])
def test_attention_benchmark_size_sampled_rows(causal, dt):
    """The timed shape, B 4 H 16 Sq = Sk = 4096 D 128, computed whole on the
    GPU; 256 sampled rows (every query tile's first and last row included for
    a few heads) checked against the oracle's rows, same bar as above."""
    B, H, S, D = 4, 16, 4096, 128
    Q, K, V = make_qkv(B, H, S, S, D, dt, seed=11)
    scale = 1.0 / math.sqrt(D)
    O, lse = run_attention(Q, K, V, dt, causal, scale)
    rng = np.random.default_rng(12)
    bh = np.concatenate([np.repeat([0, 37, 63], 2 * (S // 128)), rng.integers(0, B * H, 64)])
    edge = np.tile(np.concatenate([np.arange(0, S, 128), np.arange(127, S, 128)]), 3)
    qi = np.concatenate([edge, rng.integers(0, S, 64)])
    ref, ref_lse = oracle.attention(Q, K, V, dt, causal, scale, rows=(bh, qi))
    got = wl.bits_to_float32(O.reshape(B * H, S, D)[bh, qi], dt).astype(np.float64)
    u = 2.0 ** -9 if dt == wl.BF16 else 2.0 ** -12
    bound = 2 * u * (weighted_abs_rows(Q, K, V, dt, causal, scale, bh, qi) + np.abs(ref)) \
        + 0.5 * ulp(np.abs(ref), dt) + 1e-7
    assert np.all(np.abs(got - ref) <= bound), (np.abs(got - ref) - bound).max()
    l_got = lse.reshape(B * H, S)[bh, qi]
    assert np.all(np.abs(l_got - ref_lse) <= 1e-4 * (1 + np.abs(ref_lse)))
