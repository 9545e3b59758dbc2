"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.  Bar: relative Frobenius error <= 2e-3 and
|C - ref| <= 1e-2 |ref| + 1e-2 elementwise; on the small cases also at most
the fp32-accumulation error bound plus half an ulp of the output type."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
import workloads as wl  # noqa: E402
from gpu_util import accumulation_bound, compare, compare_f32, run_library, to_device  # noqa: E402

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def tg():
    import tensor_core_gemm_tl_b200 as m
    return m


def n_configs():
    return tg().tl_num_configs()


# every compiled kernel configuration, as the 1-based option value tl_gemm_ex takes
ALL_CONFIGS = list(range(1, n_configs() + 1))


def inputs(M, N, K, dt, epi, seed=0):
    w = wl.custom("t", M, N, K, dt, epi)
    return wl.make_inputs(w, seed)


# ------------------------------------------------------------------ layout probes
@pytest.mark.parametrize("config", ALL_CONFIGS)
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
def test_layout_probe_one_hot(config, dt):
    """A has one 1 per row (row i picks k(i)); B[k, j] encodes (k, j) as a small
    integer, so C[i, j] must equal B[k(i), j] exactly: any swizzle, descriptor
    or TMEM lane/column mistake shows as a wrong code."""
    M, N, K = 384, 320, 192
    kk = (np.arange(M) * 37 + 5) % K
    A = np.zeros((M, K), np.float32)
    A[np.arange(M), kk] = 1.0
    if dt == wl.F16:
        code = (np.arange(K)[:, None] % 32) * 32 + (np.arange(N)[None, :] % 32)
    else:
        code = (np.arange(K)[:, None] % 16) * 16 + (np.arange(N)[None, :] % 16)
    Ab = wl.round_to_bits(A, dt)
    Bb = wl.round_to_bits(code.astype(np.float32), dt)
    C = run_library(Ab, Bb, None, dt, wl.EPI_NONE, config=config)
    got = wl.bits_to_float32(C, dt)
    assert np.array_equal(got, code[kk, :].astype(np.float32))


@pytest.mark.parametrize("config", ALL_CONFIGS)
def test_identity_gives_B(config):
    n, N = 256, 384
    A = wl.round_to_bits(np.eye(n, dtype=np.float32), wl.BF16)
    _, B, _ = inputs(n, N, n, wl.BF16, 0, seed=3)
    C = run_library(A, B, None, wl.BF16, wl.EPI_NONE, config=config)
    assert np.array_equal(C, B)


# ------------------------------------------------------------------ small shapes vs the oracle
SHAPES = [
    (128, 256, 64),      # one tile, one k block
    (256, 512, 256),     # several tiles, several k blocks
    (300, 520, 200),     # ragged M, N, K tails
    (1, 1, 1),
    (15, 16, 63),
    (16, 63, 64),
    (63, 64, 65),
    (65, 127, 128),
    (127, 129, 255),
    (129, 255, 257),
    (257, 8, 16),
    (8, 257, 129),
    (1000, 24, 8),
    (70001, 24, 72),     # many tile rows, one ragged tile column
    (8, 70001, 40),      # one ragged tile row, many tile columns
]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
@pytest.mark.parametrize("epi", [wl.EPI_NONE, wl.EPI_BIAS_GELU])
def test_small_shapes_vs_oracle(M, N, K, dt, epi):
    A, B, bias = inputs(M, N, K, dt, epi, seed=M * 7 + N * 3 + K)
    ref = oracle.gemm(A, B, bias, dt, epi)
    C = run_library(A, B, bias, dt, epi)
    compare(C, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))


@pytest.mark.parametrize("config", ALL_CONFIGS)
@pytest.mark.parametrize("epi", [wl.EPI_NONE, wl.EPI_BIAS_GELU])
def test_every_config_vs_oracle(config, epi):
    M, N, K = 700, 900, 333
    for dt in (wl.F16, wl.BF16):
        A, B, bias = inputs(M, N, K, dt, epi, seed=config)
        ref = oracle.gemm(A, B, bias, dt, epi)
        C = run_library(A, B, bias, dt, epi, config=config)
        compare(C, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))


SPLIT_CASES = [
    # (M, N, K, config, dtype, epilogue): the k-blocks of a short last round
    # are spread over the units (the split forced, whatever the cost rule
    # says); a tile shared by several units is summed by the last of them to
    # finish
    (1024, 1024, 2048, 1, wl.BF16, wl.EPI_BIAS_GELU),   # 32 tiles on 148 SMs, single CTA
    (1024, 1024, 1024, 4, wl.F16, wl.EPI_NONE),         # 16 pair tiles on 74 pairs
    (1280, 1536, 1024, 4, wl.BF16, wl.EPI_BIAS_GELU),   # 30 pair tiles
    (1024, 1280, 1536, 4, wl.F16, wl.EPI_BIAS_GELU),    # 20 pair tiles
    (2560, 640, 1024, 3, wl.BF16, wl.EPI_NONE),         # a full round, then 52 tiles
    (1000, 1000, 2000, 1, wl.F16, wl.EPI_BIAS_GELU),    # ragged M, N tails
    (1001, 999, 2051, 4, wl.BF16, wl.EPI_BIAS_GELU),    # padded A and B, element stores
    (128, 4096, 4096, 2, wl.BF16, wl.EPI_BIAS_GELU),    # skinny: 32 tiles over 64 SMs
    (4000, 3000, 2050, 4, wl.BF16, wl.EPI_NONE),        # the ragged workload's shape: 44 tiles in the last round
]


@pytest.mark.parametrize("M,N,K,config,dt,epi", SPLIT_CASES)
def test_split_tiles_vs_oracle(M, N, K, config, dt, epi):
    import tensor_core_gemm_tl_b200 as m
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    p = m.plan(M, N, K, dt, "bias_gelu" if epi else None, num_sms=sms, config=config, force_split=True)
    A, B, bias = inputs(M, N, K, dt, epi, seed=M + N + K)
    ref = oracle.gemm(A, B, bias, dt, epi)
    C1 = run_library(A, B, bias, dt, epi, config=config, force_split=True)
    compare(C1, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))
    C2 = run_library(A, B, bias, dt, epi, config=config, force_split=True)
    assert np.array_equal(C1, C2), "split tiles must be bit-reproducible"
    assert p["split"] > 1 or sms != 148


@pytest.mark.parametrize("offsets", [(1, 0, 0, 0), (0, 3, 0, 0), (0, 0, 1, 0), (0, 0, 0, 5), (2, 1, 3, 7)])
def test_unaligned_bases(offsets):
    """Bases 2-byte but not 16-byte aligned: padded operand copies, the scalar
    bias path and the element-by-element store."""
    M, N, K = 200, 264, 136
    dt, epi = wl.BF16, wl.EPI_BIAS_GELU
    A, B, bias = inputs(M, N, K, dt, epi, seed=sum(offsets))
    ref = oracle.gemm(A, B, bias, dt, epi)
    C = run_library(A, B, bias, dt, epi, offsets=offsets)
    compare(C, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))


@pytest.mark.parametrize("M,N,K,offsets", [
    (333, 1002, 1030, (0, 0, 0, 0)),   # K and N even: both copies read 4-byte words
    (333, 1002, 1030, (2, 2, 0, 0)),   # bases 4 bytes past alignment: still 4-byte words
    (333, 1002, 1030, (1, 1, 0, 0)),   # bases 2 bytes past alignment: 2-byte values
    (333, 1001, 1031, (0, 0, 0, 0)),   # K and N odd: 2-byte values
])
def test_padded_copies_both_load_paths_vs_oracle(M, N, K, offsets):
    """The zero-padded copies of A and B read 4-byte words where every source
    word is 4-byte aligned and 2-byte values otherwise; both paths, for both
    operands, against the oracle."""
    m = tg()
    ptrs = tuple(256 + 2 * o for o in offsets)
    p = m.plan(M, N, K, wl.BF16, "bias_gelu", ptrs=ptrs)
    assert p["pad_a"] == 1 and p["pad_b"] == 1
    A, B, bias = inputs(M, N, K, wl.BF16, wl.EPI_BIAS_GELU, seed=M + N + K + sum(offsets))
    ref = oracle.gemm(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU)
    C = run_library(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU, offsets=offsets)
    compare(C, ref, wl.BF16, accumulation_bound(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU, ref))


def test_deterministic_bitwise():
    M, N, K = 1024, 768, 1000
    A, B, bias = inputs(M, N, K, wl.BF16, wl.EPI_BIAS_GELU, seed=42)
    c1 = run_library(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU)
    c2 = run_library(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU)
    assert np.array_equal(c1, c2)


@pytest.mark.parametrize("config", [1, 4])
def test_raster_group_changes_only_the_tile_order(config):
    """The raster group decides which tiles run together, not how a tile is
    summed: every group gives bit for bit the same C, matching the oracle."""
    import tensor_core_gemm_tl_b200 as m
    M, N, K = 1500, 1300, 700
    A, B, bias = inputs(M, N, K, wl.BF16, wl.EPI_BIAS_GELU, seed=config)
    dA, dB, db = to_device(A, wl.BF16), to_device(B, wl.BF16), to_device(bias, wl.BF16)
    ref = oracle.gemm(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU)
    outs = []
    for group in (0, 1, 3, 16, 64):
        out = m.gemm(dA, dB, db, epilogue="bias_gelu", config=config, raster_group=group, no_split=True)
        torch.cuda.synchronize()
        assert m.check_device() == 0
        outs.append(out.view(torch.int16).cpu().numpy().view(np.uint16))
        assert m.plan(M, N, K, wl.BF16, "bias_gelu", config=config, raster_group=group)["raster_group"] == \
            (min(group, m.plan(M, N, K, wl.BF16, "bias_gelu", config=config)["tiles_m"]) if group else
             m.plan(M, N, K, wl.BF16, "bias_gelu", config=config)["raster_group"])
    compare(outs[0], ref, wl.BF16, accumulation_bound(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU, ref))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_epilogue_matches_plain_plus_gelu_structure():
    """Fused result vs the oracle's epilogue applied to the oracle's plain
    product -- and the plain path from the same call site."""
    M, N, K = 256, 384, 512
    dt = wl.F16
    A, B, bias = inputs(M, N, K, dt, wl.EPI_BIAS_GELU, seed=9)
    plain = run_library(A, B, None, dt, wl.EPI_NONE)
    fused = run_library(A, B, bias, dt, wl.EPI_BIAS_GELU)
    rp = oracle.gemm(A, B, None, dt, wl.EPI_NONE)
    rf = oracle.gemm(A, B, bias, dt, wl.EPI_BIAS_GELU)
    compare(plain, rp, dt, accumulation_bound(A, B, None, dt, wl.EPI_NONE, rp))
    compare(fused, rf, dt, accumulation_bound(A, B, bias, dt, wl.EPI_BIAS_GELU, rf))


# ------------------------------------------------------------------ B given transposed, epilogue variants
@pytest.mark.parametrize("config", ALL_CONFIGS)
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
def test_transposed_b_layout_probe(config, dt):
    """B handed over as N x K (K-major): the one-hot layout probe again."""
    M, N, K = 384, 320, 192
    kk = (np.arange(M) * 37 + 5) % K
    A = np.zeros((M, K), np.float32)
    A[np.arange(M), kk] = 1.0
    code = (np.arange(K)[:, None] % 16) * 16 + (np.arange(N)[None, :] % 16)
    Ab = wl.round_to_bits(A, dt)
    Bb = wl.round_to_bits(code.astype(np.float32), dt)
    C = run_library(Ab, Bb, None, dt, wl.EPI_NONE, config=config, b_transposed=True)
    assert np.array_equal(wl.bits_to_float32(C, dt), code[kk, :].astype(np.float32))


@pytest.mark.parametrize("config", ALL_CONFIGS)
@pytest.mark.parametrize("M,N,K", [(700, 900, 336), (300, 1001, 2050), (129, 255, 64)])
def test_transposed_b_vs_oracle(config, M, N, K):
    dt, epi = wl.BF16, wl.EPI_BIAS_GELU
    A, B, bias = inputs(M, N, K, dt, epi, seed=M + config)
    ref = oracle.gemm(A, B, bias, dt, epi)
    C = run_library(A, B, bias, dt, epi, config=config, b_transposed=True)
    compare(C, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))


@pytest.mark.parametrize("epi", [wl.EPI_BIAS, wl.EPI_GELU])
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (300, 520, 200), (4096, 1024, 512)])
def test_bias_only_and_gelu_only_vs_oracle(epi, dt, M, N, K):
    A, B, bias = inputs(M, N, K, dt, epi, seed=K + epi)
    ref = oracle.gemm(A, B, bias, dt, epi)
    C = run_library(A, B, bias, dt, epi)
    compare(C, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))


TANH_F32_SHAPES = [(256, 512, 256), (300, 520, 200), (129, 1001, 2050), (4096, 1024, 512)]


@pytest.mark.parametrize("epi", [wl.EPI_BIAS_GELU_TANH, wl.EPI_GELU_TANH])
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
@pytest.mark.parametrize("M,N,K", TANH_F32_SHAPES)
def test_tanh_gelu_epilogues_vs_oracle(epi, dt, M, N, K):
    A, B, bias = inputs(M, N, K, dt, epi, seed=K + epi)
    ref = oracle.gemm(A, B, bias, dt, epi)
    C = run_library(A, B, bias, dt, epi)
    compare(C, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))


@pytest.mark.parametrize("epi", [wl.EPI_NONE, wl.EPI_BIAS_GELU, wl.EPI_BIAS, wl.EPI_GELU, wl.EPI_BIAS_GELU_TANH])
@pytest.mark.parametrize("dt", [wl.F16, wl.BF16])
@pytest.mark.parametrize("M,N,K", TANH_F32_SHAPES)
def test_float32_output_vs_oracle(epi, dt, M, N, K):
    """C in float32: the epilogue's fp32 value, never rounded to 16 bits (N = 1001
    takes the element-store tail, the others the vector stores)."""
    A, B, bias = inputs(M, N, K, dt, epi, seed=M + epi)
    ref = oracle.gemm(A, B, bias, dt, epi)
    C = run_library(A, B, bias, dt, epi, out_f32=True)
    compare_f32(C, ref, accumulation_bound(A, B, bias, dt, epi, ref, out_f32=True))


@pytest.mark.parametrize("config", ALL_CONFIGS)
def test_float32_output_every_config_and_unaligned(config):
    M, N, K = 520, 700, 264
    dt, epi = wl.BF16, wl.EPI_BIAS_GELU
    A, B, bias = inputs(M, N, K, dt, epi, seed=config)
    ref = oracle.gemm(A, B, bias, dt, epi)
    bound = accumulation_bound(A, B, bias, dt, epi, ref, out_f32=True)
    compare_f32(run_library(A, B, bias, dt, epi, config=config, out_f32=True), ref, bound)
    # C's base 4-byte but not 16-byte aligned: element stores throughout
    compare_f32(run_library(A, B, bias, dt, epi, config=config, out_f32=True, offsets=(0, 0, 0, 1)), ref, bound)


def test_float32_output_is_the_unrounded_16bit_result():
    """Rounding the float32 C once to the input type gives the 16-bit C bit for
    bit (the same accumulator, the same epilogue, one rounding moved out)."""
    M, N, K = 384, 512, 320
    for dt in (wl.F16, wl.BF16):
        for epi in (wl.EPI_NONE, wl.EPI_BIAS_GELU, wl.EPI_GELU_TANH):
            A, B, bias = inputs(M, N, K, dt, epi, seed=3)
            C16 = run_library(A, B, bias, dt, epi)
            C32 = run_library(A, B, bias, dt, epi, out_f32=True)
            assert np.array_equal(wl.round_to_bits(C32, dt), C16), (dt, epi)


# ------------------------------------------------------------------ the named workloads
def _sample_rows(M, n, rng):
    rows = {0, M - 1, M // 2}
    for t in (127, 128, 129, 255, 256):
        if t < M:
            rows.add(t)
    rows.update(int(r) for r in rng.integers(0, M, n))
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_workload_sampled_vs_oracle(name):
    """Every named workload at full size in the launch configuration the
    benchmark times (the library's choice): whole rows of C sampled and
    compared with the oracle's rows (the 256^3 case in full)."""
    w = wl.WORKLOADS[name]
    A, B, bias = wl.make_inputs(w, 0)
    C = run_library(A, B, bias, w.dtype, w.epi)
    if w.M * w.N * w.K <= 1 << 28:
        ref = oracle.gemm(A, B, bias, w.dtype, w.epi)
        compare(C, ref, w.dtype, accumulation_bound(A, B, bias, w.dtype, w.epi, ref))
        return
    rng = np.random.default_rng(1)
    budget_rows = max(8, int(4e9 // (2 * w.N * w.K)))
    rows = _sample_rows(w.M, min(48, budget_rows), rng)
    ref = oracle.gemm(A, B, bias, w.dtype, w.epi, rows=rows)
    compare(C[rows], ref, w.dtype, accumulation_bound(A, B, bias, w.dtype, w.epi, ref, rows=rows))
    # and scattered single elements over the whole of C
    ii = rng.integers(0, w.M, 2000)
    jj = rng.integers(0, w.N, 2000)
    refp = oracle.gemm_points(A, B, bias, w.dtype, w.epi, ii, jj)
    compare(C[ii, jj], refp, w.dtype, accumulation_bound(A, B, bias, w.dtype, w.epi, refp, points=(ii, jj)))


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_reports_timeout_and_context_survives():
    """The copy warp skips its first stage without issuing the copy: the MMA
    warp's bounded wait runs out, the kernel records it and returns.  The
    status is read on the host; the next call on the same context is right."""
    import tensor_core_gemm_tl_b200 as m
    M, N, K = 256, 256, 256
    A, B, bias = inputs(M, N, K, wl.F16, 0, seed=5)
    dA, dB = to_device(A, wl.F16), to_device(B, wl.F16)
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    opt = m.Options(config=0, inject_fault=1, timeout_ns=200_000_000)
    st = m.tl_gemm_ex(dA.data_ptr(), dB.data_ptr(), 0, out.data_ptr(), M, N, K, wl.F16, 0,
                      torch.cuda.current_stream().cuda_stream, opt)
    assert st == 0
    st, word = m.tl_check_device(torch.cuda.current_stream().cuda_stream)
    assert st == int(m.Status.DEVICE_TIMEOUT)
    assert word & 2  # the MMA warp's wait on data gave up
    assert not (word & 16)  # and every issued copy / MMA drained in time
    st, word = m.tl_check_device(torch.cuda.current_stream().cuda_stream)
    assert st == 0 and word == 0  # the word was cleared
    C = run_library(A, B, None, wl.F16, 0)
    ref = oracle.gemm(A, B, None, wl.F16, 0)
    compare(C, ref, wl.F16, accumulation_bound(A, B, None, wl.F16, 0, ref))


@pytest.mark.parametrize("config", ALL_CONFIGS)
def test_fault_hook_on_every_config_drains_and_context_survives(config):
    """Every producer (with a CTA pair, both CTAs' producers) skips the same
    stage without issuing its copies: the MMA warp's wait on that stage runs
    out, the kernel records it, drains the copies it did issue -- the even
    CTA of a pair waits on its barriers for both CTAs' copies -- frees Tensor
    Memory and returns.  Bit 1 is set and the drain bit is clear; the next
    calls on the same context, with and without a split last round, are
    right."""
    import tensor_core_gemm_tl_b200 as m
    stream = torch.cuda.current_stream().cuda_stream
    for M, N, K in ((512, 512, 1024), (1024, 1024, 2048)):
        A, B, bias = inputs(M, N, K, wl.BF16, wl.EPI_BIAS_GELU, seed=config)
        dA, dB, db = to_device(A, wl.BF16), to_device(B, wl.BF16), to_device(bias, wl.BF16)
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        opt = m.Options(config=config, inject_fault=1, timeout_ns=100_000_000)
        st = m.tl_gemm_ex(dA.data_ptr(), dB.data_ptr(), db.data_ptr(), out.data_ptr(), M, N, K, wl.BF16,
                          wl.EPI_BIAS_GELU, stream, opt)
        assert st == 0
        st, word = m.tl_check_device(stream)
        assert st == int(m.Status.DEVICE_TIMEOUT)
        assert word & 2, word          # the MMA warp's wait on data gave up
        assert not (word & 16), word   # every issued copy and MMA drained in time
        assert not (word & 128), word
        ref = oracle.gemm(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU)
        C = run_library(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU, config=config)
        compare(C, ref, wl.BF16, accumulation_bound(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU, ref))


def test_host_side_encode_failure_is_reported_and_nothing_runs():
    """The host treats A's tensor-map encode as failed (test hook 2): the call
    returns TL_ERR_CUDA before any kernel is launched, C is untouched, no device
    error is recorded, and the next call on the same context is right."""
    import tensor_core_gemm_tl_b200 as m
    M, N, K = 256, 384, 320
    A, B, bias = inputs(M, N, K, wl.BF16, wl.EPI_BIAS_GELU, seed=9)
    dA, dB, dbias = to_device(A, wl.BF16), to_device(B, wl.BF16), to_device(bias, wl.BF16)
    out = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = m.tl_gemm_ex(dA.data_ptr(), dB.data_ptr(), dbias.data_ptr(), out.data_ptr(), M, N, K, wl.BF16,
                      wl.EPI_BIAS_GELU, stream, m.Options(inject_fault=2))
    assert st == int(m.Status.CUDA)
    st, word = m.tl_check_device(stream)
    assert st == 0 and word == 0
    assert bool(torch.all(out == 7.0))
    C = run_library(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU)
    ref = oracle.gemm(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU)
    compare(C, ref, wl.BF16, accumulation_bound(A, B, bias, wl.BF16, wl.EPI_BIAS_GELU, ref))


# ------------------------------------------------------------------ concurrent callers
def test_split_gemms_on_concurrent_streams_never_wait_on_each_other():
    """No part of a split tile waits for another unit, so GEMMs whose last
    round is split can share the GPU with anything: two split GEMMs launched
    together on two streams, a split GEMM launched while a long plain GEMM
    holds every SM, and a split GEMM through tl_gemm_noalloc beside one
    through tl_gemm.  Each returns TL_OK with no device error, matches the
    oracle, and equals bit for bit the same call made alone."""
    import tensor_core_gemm_tl_b200 as m
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cases = [(1024, 1024, 2048, 1, wl.BF16, wl.EPI_BIAS_GELU), (1280, 1536, 1024, 4, wl.F16, wl.EPI_NONE)]
    bufs = []
    for M, N, K, config, dt, epi in cases:
        assert m.plan(M, N, K, dt, "bias_gelu" if epi else None, num_sms=sms, config=config,
                      force_split=True)["split"] > 1
        A, B, bias = inputs(M, N, K, dt, epi, seed=M + K)
        dA, dB = to_device(A, dt), to_device(B, dt)
        db = to_device(bias, dt) if bias is not None else None
        ref = oracle.gemm(A, B, bias, dt, epi)
        alone = run_library(A, B, bias, dt, epi, config=config, force_split=True)
        compare(alone, ref, dt, accumulation_bound(A, B, bias, dt, epi, ref))
        bufs.append((M, N, K, config, dt, epi, dA, dB, db, alone))
    big = torch.randn(8192, 8192, device="cuda").to(torch.bfloat16)
    big_out = torch.empty_like(big)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()

    def launch(case, stream, entry="ex"):
        M, N, K, config, dt, epi, dA, dB, db, _ = case
        out = torch.empty((M, N), dtype=torch.float16 if dt == wl.F16 else torch.bfloat16, device="cuda")
        bp = db.data_ptr() if db is not None else 0
        if entry == "noalloc":
            st = m.tl_gemm_noalloc(dA.data_ptr(), dB.data_ptr(), bp, out.data_ptr(), M, N, K, dt, epi,
                                   stream.cuda_stream)
        else:
            st = m.tl_gemm_ex(dA.data_ptr(), dB.data_ptr(), bp, out.data_ptr(), M, N, K, dt, epi, stream.cuda_stream,
                              m.Options(config=config, force_split=1))
        assert st == 0, m.tl_status_string(st)
        return out

    def bits(t):
        return t.view(torch.int16).cpu().numpy().view(np.uint16)

    for rep in range(3):
        torch.cuda.synchronize()
        # two split GEMMs at once
        o1, o2 = launch(bufs[0], s1), launch(bufs[1], s2)
        # a split GEMM behind a long GEMM that fills every SM
        with torch.cuda.stream(s1):
            t = tg()
            t.gemm(big, big, out=big_out, stream=s1)
        o3 = launch(bufs[0], s2)
        # the allocation-free entry point beside tl_gemm (separate workspaces)
        M, N, K, config, dt, epi = cases[0][:6]
        if m.plan(M, N, K, dt, "bias_gelu", num_sms=sms)["split"] > 1:
            o4 = launch(bufs[0], s1, "noalloc")
            o5 = launch(bufs[0], s2, "ex")
        else:
            o4 = o5 = None
        torch.cuda.synchronize()
        assert t.check_device() == 0
        assert np.array_equal(bits(o1), bufs[0][-1]) and np.array_equal(bits(o3), bufs[0][-1])
        assert np.array_equal(bits(o2), bufs[1][-1])
        if o4 is not None:
            assert np.array_equal(bits(o5), bufs[0][-1])
            ref = oracle.gemm(*inputs(M, N, K, dt, epi, seed=M + K), dt, epi)
            compare(bits(o4), ref, dt)



def test_concurrent_calls_from_threads_on_their_own_streams():
    """Eight threads call the library at once, each on a stream of its own
    (ctypes releases the GIL for every call): GEMMs that take the padded-copy
    path and the split last round (both with workspace from the stream-ordered
    pool) and the plain path, attention and row softmax.  Every output equals,
    bit for bit, the same call made alone beforehand on one thread."""
    from concurrent.futures import ThreadPoolExecutor
    t = tg()
    assert t.plan(16384, 1024, 8192, dtype=1)["split"] > 1 and t.plan(4000, 3000, 2050, dtype=1)["pad_a"]
    g = torch.Generator(device="cuda").manual_seed(7)

    def rnd(*shape):
        return torch.randn(*shape, device="cuda", generator=g).to(torch.bfloat16)

    jobs = {
        "split": (rnd(16384, 8192), rnd(8192, 1024), None, None),
        "padded": (rnd(4000, 2050), rnd(2050, 3000), rnd(3000), "bias_gelu"),
        "plain": (rnd(1024, 768), rnd(768, 2048), rnd(2048), "bias"),
    }
    qkv = [rnd(2, 4, 700, 128) for _ in range(3)]
    xs = rnd(333, 50257)

    def run(name, stream):
        if name == "attention":
            return t.attention(*qkv, causal=True, stream=stream)
        if name == "softmax":
            return t.softmax(xs, stream=stream)
        A, B, bias, epi = jobs[name]
        return t.gemm(A, B, bias, epilogue=epi, stream=stream)

    names = list(jobs) + ["attention", "softmax"]
    torch.cuda.synchronize()
    alone = {n: run(n, torch.cuda.current_stream()).view(torch.int16).cpu() for n in names}
    assert t.check_device() == 0

    def worker(idx):
        s = torch.cuda.Stream()
        order = names[idx % len(names):] + names[:idx % len(names)]
        with torch.cuda.stream(s):
            outs = {n: run(n, s) for n in order for _ in range(2)}
        s.synchronize()
        return {n: o.view(torch.int16).cpu() for n, o in outs.items()}

    with ThreadPoolExecutor(max_workers=8) as pool:
        results = list(pool.map(worker, range(8)))
    torch.cuda.synchronize()
    assert t.check_device() == 0
    for res in results:
        for n in names:
            assert torch.equal(res[n], alone[n]), n
