"""The C-ABI library on the CPU: it loads, exports every symbol the header
declares, validates arguments before touching a GPU, and plans launches
(configuration, grid, padding, store path) as documented."""
import os
import re

import numpy as np
import pytest

import tensor_core_gemm_tl_b200 as tg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tl_gemm.h")
P = 1 << 20  # a fake, 256-byte aligned "device pointer" (never dereferenced on the CPU)


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TL_API\s+[\w\s\*]+?\b(tl_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert {"tl_gemm", "tl_gemm_ex", "tl_check_device", "tl_gemm_plan", "tl_num_configs",
            "tl_config_name", "tl_status_string", "tl_version"} <= set(names)


def test_library_exports_every_declared_symbol():
    lib = tg._binding._lib
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in tg.SIGNATURES, f"binding lacks {name}"


def test_version_and_strings():
    declared = int(re.search(r"#define TL_VERSION (\d+)", open(HEADER).read()).group(1))
    assert tg.tl_version() == declared
    for s in tg.Status:
        assert tg.tl_status_string(int(s)) == "TL_" + ("OK" if s.name == "OK" else "ERR_" + s.name)
    assert tg.tl_status_string(99) == "TL_ERR_UNKNOWN"
    n = tg.tl_num_configs()
    assert n >= 3
    names = tg.configs()
    assert all(re.fullmatch(r"bm\d+_bn\d+_bk\d+_s\d+(_pair)?", x) for x in names)
    assert tg.tl_config_name(n) is None and tg.tl_config_name(-1) is None


@pytest.mark.parametrize("args,status", [
    (dict(A=0), tg.Status.INVALID_ARG),
    (dict(B=0), tg.Status.INVALID_ARG),
    (dict(C=0), tg.Status.INVALID_ARG),
    (dict(M=0), tg.Status.INVALID_ARG),
    (dict(N=-1), tg.Status.INVALID_ARG),
    (dict(K=0), tg.Status.INVALID_ARG),
    (dict(dtype=2), tg.Status.INVALID_ARG),
    (dict(epi=6), tg.Status.INVALID_ARG),
    (dict(epi=-1), tg.Status.INVALID_ARG),
    (dict(epi=1, bias=0), tg.Status.INVALID_ARG),
    (dict(epi=2, bias=0), tg.Status.INVALID_ARG),
    (dict(epi=4, bias=0), tg.Status.INVALID_ARG),
    (dict(epi=4, bias=P + 1), tg.Status.MISALIGNED),
    (dict(epi=2, bias=P + 1), tg.Status.MISALIGNED),
    (dict(M=1 << 31), tg.Status.UNSUPPORTED),
    (dict(K=1 << 40), tg.Status.UNSUPPORTED),
    (dict(A=P + 1), tg.Status.MISALIGNED),
    (dict(C=P + 3), tg.Status.MISALIGNED),
    (dict(epi=1, bias=P + 1), tg.Status.MISALIGNED),
])
def test_validation_before_any_cuda_call(args, status):
    a = dict(A=P, B=P, bias=0, C=P, M=64, N=64, K=64, dtype=0, epi=0)
    a.update(args)
    st = tg.tl_gemm(a["A"], a["B"], a["bias"], a["C"], a["M"], a["N"], a["K"], a["dtype"], a["epi"], 0)
    assert st == status
    st2, _ = tg.tl_gemm_plan(a["A"], a["B"], a["bias"], a["C"], a["M"], a["N"], a["K"], a["dtype"],
                             a["epi"], 148)
    assert st2 == status


def test_options_validation():
    bad = tg.Options(config=tg.tl_num_configs() + 1)
    assert tg.tl_gemm_ex(P, P, 0, P, 8, 8, 8, 0, 0, 0, bad) == tg.Status.INVALID_ARG
    bad = tg.Options(config=-1)
    assert tg.tl_gemm_ex(P, P, 0, P, 8, 8, 8, 0, 0, 0, bad) == tg.Status.INVALID_ARG
    bad = tg.Options(inject_fault=3)
    assert tg.tl_gemm_ex(P, P, 0, P, 8, 8, 8, 0, 0, 0, bad) == tg.Status.INVALID_ARG


@pytest.mark.skipif(os.environ.get("CUDA_VISIBLE_DEVICES") is None and __import__("torch").cuda.is_available(),
                    reason="only meaningful without a GPU")
def test_no_device_is_a_cuda_error_not_a_crash():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert tg.tl_gemm(P, P, 0, P, 64, 64, 64, 0, 0, 0) == tg.Status.CUDA


def test_plan_aligned_headline_shape():
    p = tg.plan(4096, 4096, 4096, tg.TL_F16, None, num_sms=148)
    assert p["pad_a"] == 0 and p["pad_b"] == 0 and p["direct_store"] == 0
    assert (p["workspace_bytes"] == 0) == (p["split"] == 1)  # only split tiles need a workspace
    assert p["tiles_m"] == 4096 // p["block_m"] and p["tiles_n"] == 4096 // p["block_n"]
    assert p["grid"] == min(148 // p["cluster_ctas"], p["tiles_m"] * p["tiles_n"]) * p["cluster_ctas"]
    assert p["smem_bytes"] <= 232448


def test_plan_grid_never_exceeds_tiles():
    p = tg.plan(100, 60, 30, tg.TL_BF16, None, num_sms=148)
    assert p["tiles_m"] == 1 and p["tiles_n"] == 1 and p["grid"] == p["cluster_ctas"]


def test_plan_unaligned_k_pads_A_only():
    M, N, K = 4000, 3000, 2050
    p = tg.plan(M, N, K, tg.TL_BF16, "bias_gelu", num_sms=148)
    assert p["pad_a"] == 1 and p["pad_b"] == 0 and p["direct_store"] == 0
    assert p["workspace_bytes"] == ((M * 2112 * 2 + 255) // 256) * 256  # rows of whole 128-byte lines


def test_plan_unaligned_n_pads_B_and_stores_directly():
    M, N, K = 300, 1001, 64
    p = tg.plan(M, N, K, tg.TL_F16, None, num_sms=148)
    assert p["pad_a"] == 0 and p["pad_b"] == 1 and p["direct_store"] == 1
    assert p["workspace_bytes"] == ((K * 1024 * 2 + 255) // 256) * 256


def test_plan_misaligned_bases():
    # 2-byte aligned but not 16-byte aligned bases take the padded / direct paths
    p = tg.plan(256, 256, 256, tg.TL_F16, None, num_sms=148, ptrs=(P + 2, P + 6, 0, P + 8))
    assert p["pad_a"] == 1 and p["pad_b"] == 1 and p["direct_store"] == 1


def test_plan_forced_config():
    for k in range(1, tg.tl_num_configs() + 1):
        p = tg.plan(4096, 4096, 4096, tg.TL_F16, None, num_sms=148, config=k)
        assert p["config"] == k - 1
        assert p["config_name"] == tg.tl_config_name(k - 1)
        pair = p["config_name"].endswith("_pair")
        assert p["cluster_ctas"] == (2 if pair else 1)
        assert p["grid"] % p["cluster_ctas"] == 0 and p["grid"] <= 148


def test_fault_hook_is_accepted_on_every_config():
    # single CTAs and CTA pairs alike: with a pair, both CTAs skip the same stage
    for k in range(1, tg.tl_num_configs() + 1):
        opt = tg.Options(config=k, inject_fault=1)
        st, p = tg.tl_gemm_plan(P, P, 0, P, 512, 512, 512, 0, 0, 148, opt)
        assert st == 0 and p.config == k - 1
        assert p.cluster_ctas == (2 if tg.tl_config_name(k - 1).endswith("_pair") else 1)


def test_plan_skinny_prefers_narrow_tiles():
    # 128 x 16384: a 128 x 256 tiling leaves most of 148 SMs idle
    wide = tg.plan(128, 16384, 4096, tg.TL_BF16, None, num_sms=148, config=1)
    chosen = tg.plan(128, 16384, 4096, tg.TL_BF16, None, num_sms=148)
    assert wide["tiles_m"] * wide["tiles_n"] < 148
    assert chosen["tiles_m"] * chosen["tiles_n"] > wide["tiles_m"] * wide["tiles_n"]


def test_torch_wrapper_rejects_bad_tensors():
    import torch
    A = torch.zeros(4, 4, dtype=torch.float16)
    with pytest.raises(ValueError):
        tg.gemm(A, A)  # CPU tensors
    with pytest.raises(ValueError):
        tg.gemm(A, torch.zeros(5, 4, dtype=torch.float16))
    with pytest.raises(ValueError):
        tg._epi_code("relu")


class _FakeCuda:
    """Stands in for a CUDA tensor on a machine without one: it carries what
    the binding's checks read, and fails the test if a pointer is taken."""

    def __init__(self, shape, dtype, device="cuda:0", contiguous=True):
        import torch
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self.is_cuda = self.device.type == "cuda"
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)

    def numel(self):
        return int(np.prod(self.shape))

    def data_ptr(self):
        raise AssertionError("a pointer was taken from a tensor that should have been rejected")


def _bad_tensor_cases():
    import torch
    bf, f32 = torch.bfloat16, torch.float32
    F = _FakeCuda
    cpu = lambda shape, dt: torch.zeros(shape, dtype=dt)  # noqa: E731
    q = lambda: F((1, 2, 128, 64), bf)  # noqa: E731
    x = lambda: F((8, 256), bf)  # noqa: E731
    v = lambda: F((1000,), f32)  # noqa: E731
    A, B = (lambda: F((64, 32), bf)), (lambda: F((32, 48), bf))  # noqa: E731
    return [
        # attention: out / lse on the host, on another device, of the wrong shape, dtype or layout
        ("attention", lambda: tg.attention(q(), q(), q(), out=cpu((1, 2, 128, 64), bf))),
        ("attention", lambda: tg.attention(q(), q(), q(), out=F((1, 2, 128, 64), bf, "cuda:1"))),
        ("attention", lambda: tg.attention(q(), q(), q(), out=F((1, 2, 128, 64), bf, contiguous=False))),
        ("attention", lambda: tg.attention(q(), q(), q(), lse=cpu((1, 2, 128), f32))),
        ("attention", lambda: tg.attention(q(), q(), q(), lse=F((1, 2, 128), bf))),
        ("attention", lambda: tg.attention(q(), q(), q(), lse=F((1, 2, 127), f32))),
        ("attention", lambda: tg.attention(q(), q(), q(), lse=F((1, 2, 128), f32, contiguous=False))),
        ("attention", lambda: tg.attention(q(), F((1, 2, 128, 64), bf, "cuda:1"), q())),
        # softmax: out on the host or elsewhere
        ("softmax", lambda: tg.softmax(x(), out=cpu((8, 256), bf))),
        ("softmax", lambda: tg.softmax(x(), out=F((8, 256), bf, "cuda:1"))),
        ("softmax", lambda: tg.softmax(x(), out=F((8, 256), bf, contiguous=False))),
        ("softmax", lambda: tg.softmax(x(), out=F((8, 255), bf))),
        # vector add: b and out on the host, elsewhere, strided, or of another shape
        ("vector_add", lambda: tg.vector_add(v(), cpu((1000,), f32))),
        ("vector_add", lambda: tg.vector_add(v(), F((1000,), f32, "cuda:1"))),
        ("vector_add", lambda: tg.vector_add(v(), F((1000,), f32, contiguous=False))),
        ("vector_add", lambda: tg.vector_add(F((1000,), f32, contiguous=False), v())),
        ("vector_add", lambda: tg.vector_add(v(), v(), out=cpu((1000,), f32))),
        ("vector_add", lambda: tg.vector_add(v(), v(), out=F((999,), f32))),
        ("vector_add", lambda: tg.vector_add(v(), v(), out=F((1000,), f32, contiguous=False))),
        # GEMM: B, bias and out on the host or another device
        ("gemm", lambda: tg.gemm(A(), F((32, 48), bf, "cuda:1"))),
        ("gemm", lambda: tg.gemm(A(), B(), cpu((48,), bf))),
        ("gemm", lambda: tg.gemm(A(), B(), F((48,), bf, "cuda:1"))),
        ("gemm", lambda: tg.gemm(A(), B(), out=cpu((64, 48), bf))),
        ("gemm", lambda: tg.gemm(A(), B(), out=F((64, 48), bf, "cuda:1"))),
    ]


@pytest.mark.parametrize("case", range(24))
def test_binding_rejects_host_and_foreign_tensors_before_any_launch(case, monkeypatch):
    cases = _bad_tensor_cases()
    assert len(cases) == 24
    _, call = cases[case]

    def no_launch(*a, **k):
        raise AssertionError("the C ABI was called with a tensor the binding should have rejected")

    for name in ("tl_gemm", "tl_gemm_ex", "tl_attention_fwd", "tl_softmax_rows", "tl_vector_add"):
        monkeypatch.setattr(tg, name, no_launch)
    with pytest.raises(ValueError):
        call()


@pytest.mark.parametrize("M,N,K,config,dtype,split,full", [
    # the cost rule: split only when the k-blocks saved exceed the reduction's round trips
    (4096, 4096, 4096, 4, 1, True, 222),    # 256 pair tiles on 74 pairs: 3 rounds + 34 tiles over 68 pairs
    (4096, 4096, 4096, 1, 1, True, 444),    # 512 single-CTA tiles on 148: 68 left over
    (1024, 1024, 2048, 1, 1, True, 0),      # 32 tiles, 2 units each
    (1024, 1024, 1024, 4, 1, False, 16),    # 16 pair tiles of 16 k-blocks: too little to save
    (2560, 640, 1024, 3, 1, False, 200),    # 200 tiles of 128 x 64, 16 k-blocks each
    (128, 16384, 4096, 2, 1, False, 128),   # the skinny shape: 128 tiles on 148 SMs
    (4000, 3000, 2050, 4, 1, False, 192),   # the ragged shape: 33 k-blocks per tile
    (8192, 16384, 4096, 4, 1, True, 1998),  # 2048 pair tiles = 27 rounds of 74 + 50
    (700, 900, 333, 4, 1, False, 12),       # too few k-blocks to split
    (16384, 1024, 8192, 4, 1, True, 222),   # the tall shape
])
def test_plan_splits_only_a_short_last_round(M, N, K, config, dtype, split, full):
    from schedule_model import check_schedule
    p = tg.plan(M, N, K, dtype, None, num_sms=148, config=config)
    tiles = p["tiles_m"] * p["tiles_n"]
    assert (p["split"] > 1) == split and p["full_tiles"] == full
    parts = check_schedule(p, 148, K)
    if split:
        slabs = p["num_slots"] * p["cluster_ctas"]
        assert p["workspace_bytes"] >= slabs * 128 * p["block_n"] * 4
        assert parts <= 3 and p["tail_units"] <= 2 * (tiles - full)  # at most two units per tile on average
    else:
        assert p["workspace_bytes"] == 0 or p["pad_a"] or p["pad_b"]
    # forcing the split takes it wherever the last round is partial and K is long enough
    f = tg.plan(M, N, K, dtype, None, num_sms=148, config=config, force_split=True)
    units = 148 // f["cluster_ctas"]
    assert (f["split"] > 1) == (tiles % units != 0 and -(-K // 64) >= 8)
    check_schedule(f, 148, K)
    # and no_split never does
    n = tg.plan(M, N, K, dtype, None, num_sms=148, config=config, no_split=True)
    assert n["split"] == 1 and n["full_tiles"] == tiles and n["tail_units"] == 0


def test_split_options_are_validated():
    for bad in (tg.Options(force_split=2), tg.Options(force_split=1, no_split=1), tg.Options(raster_group=-1)):
        st, _ = tg.tl_gemm_plan(P, P, 0, P, 64, 64, 64, 0, 0, 148, bad)
        assert st == tg.Status.INVALID_ARG


def test_host_fault_hook_is_valid_and_changes_no_plan():
    # 2: the host-side hook (a refused tensor-map encode) plans like a normal call
    st, p = tg.tl_gemm_plan(P, P, 0, P, 4096, 4096, 4096, 0, 0, 148, tg.Options(inject_fault=2))
    st0, p0 = tg.tl_gemm_plan(P, P, 0, P, 4096, 4096, 4096, 0, 0, 148)
    assert st == 0 and st0 == 0 and p.config == p0.config and p.split == p0.split and p.grid == p0.grid
    assert tg.tl_gemm_ex(P, P, 0, P, 8, 8, 8, 0, 0, 0, tg.Options(inject_fault=-1)) == tg.Status.INVALID_ARG


def test_fault_hook_plans_like_a_normal_call():
    # the copy-skipping hook runs on the configuration the shape would use
    # (CTA pairs included) with the same work split
    for cfg in (0, 1, 4):
        st, p = tg.tl_gemm_plan(P, P, 0, P, 1024, 1024, 2048, 0, 0, 148, tg.Options(config=cfg, inject_fault=1))
        st0, p0 = tg.tl_gemm_plan(P, P, 0, P, 1024, 1024, 2048, 0, 0, 148, tg.Options(config=cfg))
        assert st == 0 and st0 == 0 and p.as_dict() == p0.as_dict()


def test_gelu_only_needs_no_bias_and_b_layout_is_validated():
    st, _ = tg.tl_gemm_plan(P, P, 0, P, 256, 256, 256, 0, tg.TL_EPI_GELU, 148)
    assert st == 0
    assert tg.tl_gemm_ex(P, P, 0, P, 8, 8, 8, 0, 0, 0, tg.Options(b_layout=2)) == tg.Status.INVALID_ARG


def test_tanh_epilogues_and_float32_output_options():
    # tanh GELU alone needs no bias; with bias it does
    st, _ = tg.tl_gemm_plan(P, P, 0, P, 256, 256, 256, 0, tg.TL_EPI_GELU_TANH, 148)
    assert st == 0
    st, _ = tg.tl_gemm_plan(P, P, P, P, 256, 256, 256, 1, tg.TL_EPI_BIAS_GELU_TANH, 148)
    assert st == 0
    # float32 C: 4-byte alignment, never the TMA store, same tiles and padding
    f32 = tg.Options(c_float32=1)
    st, p = tg.tl_gemm_plan(P, P, 0, P, 4096, 4096, 4096, 0, 0, 148, f32)
    assert st == 0 and p.direct_store == 1 and p.pad_a == 0 and p.pad_b == 0
    st, p16 = tg.tl_gemm_plan(P, P, 0, P, 4096, 4096, 4096, 0, 0, 148)
    assert st == 0 and p16.direct_store == 0 and p16.config == p.config and p16.grid == p.grid
    assert tg.tl_gemm_ex(P, P, 0, P + 2, 8, 8, 8, 0, 0, 0, f32) == tg.Status.MISALIGNED
    assert tg.tl_gemm_ex(P, P, 0, P, 8, 8, 8, 0, 0, 0, tg.Options(c_float32=2)) == tg.Status.INVALID_ARG
    assert tg.plan(512, 1000, 2048, tg.TL_BF16, "gelu_tanh", c_float32=True)["direct_store"] == 1


def test_plan_transposed_b_pads_on_k():
    # B given as N x K: its rows are K long, so an odd K pads B (and A), not N
    p = tg.plan(512, 1000, 2050, tg.TL_BF16, None, num_sms=148, b_transposed=True)
    assert p["pad_a"] == 1 and p["pad_b"] == 1 and p["direct_store"] == 0
    p = tg.plan(512, 1001, 2048, tg.TL_BF16, None, num_sms=148, b_transposed=True)
    assert p["pad_a"] == 0 and p["pad_b"] == 0 and p["direct_store"] == 1
    p = tg.plan(512, 1001, 2048, tg.TL_BF16, None, num_sms=148)
    assert p["pad_b"] == 1


@pytest.mark.parametrize("args,status", [
    (dict(Q=0), tg.Status.INVALID_ARG),
    (dict(O=0), tg.Status.INVALID_ARG),
    (dict(batch=0), tg.Status.INVALID_ARG),
    (dict(seq_k=0), tg.Status.INVALID_ARG),
    (dict(head_dim=96), tg.Status.UNSUPPORTED),
    (dict(head_dim=256), tg.Status.UNSUPPORTED),
    (dict(dtype=5), tg.Status.INVALID_ARG),
    (dict(scale=-1.0), tg.Status.INVALID_ARG),
    (dict(scale=float("nan")), tg.Status.INVALID_ARG),
    (dict(batch=256, heads=256), tg.Status.UNSUPPORTED),   # non-causal: batch * heads beyond 65535
    (dict(K=P + 2), tg.Status.MISALIGNED),
    (dict(lse=P + 2), tg.Status.MISALIGNED),
])
def test_attention_validation_before_any_cuda_call(args, status):
    a = dict(Q=P, K=P, V=P, O=P, lse=0, batch=1, heads=2, seq_q=64, seq_k=64, head_dim=64, dtype=0, scale=0.0)
    a.update(args)
    st = tg.tl_attention_fwd(a["Q"], a["K"], a["V"], a["O"], a["lse"], a["batch"], a["heads"], a["seq_q"],
                             a["seq_k"], a["head_dim"], a["dtype"], False, a["scale"], 0)
    assert st == status


def test_attention_causal_grid_limits():
    # causal launches put batch * heads along x (up to 2^31 - 1) and the
    # query-tile pairs along y (up to 65535)
    def st(batch, heads, seq_q):
        return tg.tl_attention_fwd(P, P, P, P, 0, batch, heads, seq_q, 64, 64, 0, True, 0.0, 0)
    assert st(1 << 16, 1 << 15, 64) == tg.Status.UNSUPPORTED
    assert st(1, 2, 65536 * 256) == tg.Status.UNSUPPORTED
    assert st(256, 256, 64) != tg.Status.UNSUPPORTED  # fine when causal (fails later only for want of a GPU)


def test_softmax_and_vector_add_validation():
    assert tg.tl_softmax_rows(0, P, 4, 4, 0, 0) == tg.Status.INVALID_ARG
    assert tg.tl_softmax_rows(P, P, 0, 4, 0, 0) == tg.Status.INVALID_ARG
    assert tg.tl_softmax_rows(P, P, 4, 0, 0, 0) == tg.Status.INVALID_ARG
    assert tg.tl_softmax_rows(P, P, 4, 4, 9, 0) == tg.Status.INVALID_ARG
    assert tg.tl_softmax_rows(P + 1, P, 4, 4, 0, 0) == tg.Status.MISALIGNED
    assert tg.tl_vector_add(P, 0, P, 4, 0) == tg.Status.INVALID_ARG
    assert tg.tl_vector_add(P, P, P, 0, 0) == tg.Status.INVALID_ARG
    assert tg.tl_vector_add(P + 2, P, P, 4, 0) == tg.Status.MISALIGNED


def test_plan_is_total_and_consistent_for_any_shape():
    """Every shape gets a configuration, and the plan is self-consistent: the
    tiles cover C, the grid is at most one unit per SM (or pair), a split
    only cuts the last round and the kernel's schedule then computes every
    k-block of every tile exactly once, the shared memory fits and the
    workspace holds the padded copies (property test over random shapes,
    dtypes, epilogues and layouts)."""
    from hypothesis import given, settings, strategies as st
    from schedule_model import check_schedule

    @settings(max_examples=400, deadline=None)
    @given(M=st.integers(1, 70000), N=st.integers(1, 70000), K=st.integers(1, 70000),
           dtype=st.sampled_from([0, 1]), epi=st.integers(0, 5), bt=st.booleans(), f32=st.booleans(),
           sms=st.sampled_from([148, 132, 8]))
    def check(M, N, K, dtype, epi, bt, f32, sms):
        bias = P if epi in (1, 2, 4) else 0
        opt = tg.Options(b_layout=int(bt), c_float32=int(f32))
        s, p = tg.tl_gemm_plan(P, P, bias, P, M, N, K, dtype, epi, sms, opt)
        assert s == 0, (M, N, K, s)
        assert 0 <= p.config < tg.tl_num_configs()
        assert p.tiles_m * p.block_m >= M and (p.tiles_m - 1) * p.block_m < M
        assert p.tiles_n * p.block_n >= N and (p.tiles_n - 1) * p.block_n < N
        tiles = p.tiles_m * p.tiles_n
        units = sms // p.cluster_ctas
        assert 1 <= p.grid // p.cluster_ctas <= min(units, max(tiles, p.tail_units))
        assert p.grid % p.cluster_ctas == 0
        assert p.split >= 1 and (p.split == 1) == (p.full_tiles == tiles)
        assert p.split == 1 or tiles - p.full_tiles < units  # only the short last round is split
        if tiles <= 20000:
            check_schedule(p.as_dict(), sms, K)  # every k-block of every tile exactly once
        assert p.smem_bytes <= 232448
        assert bool(p.direct_store) == (f32 or N % 8 != 0)  # base pointers here are 256-byte aligned
        need = 0
        if p.pad_a:
            need += M * ((K + 63) // 64 * 64) * 2
        if p.pad_b:
            rows, cols = (N, K) if bt else (K, N)
            need += rows * ((cols + 63) // 64 * 64) * 2
        assert p.workspace_bytes >= need

    check()


def test_split_schedule_covers_every_k_block_once():
    """For shapes of up to a few thousand tiles, with every configuration and
    several unit counts, the schedule the kernel derives from the plan (the
    index arithmetic of its unit_work / tail_contributors, restated in
    tests/schedule_model.py) computes every k-block of every tile exactly
    once, sums each shared tile over the units the kernel adds up, and keeps
    partial-sum slots inside the workspace."""
    from hypothesis import given, settings, strategies as st
    from schedule_model import check_schedule
    seen = {"split": 0}

    @settings(max_examples=600, deadline=None)
    @given(M=st.integers(1, 9000), N=st.integers(1, 9000), K=st.integers(1, 20000),
           config=st.integers(0, tg.tl_num_configs()), sms=st.sampled_from([148, 132, 20, 8, 2]),
           force=st.booleans())
    def check(M, N, K, config, sms, force):
        s, p = tg.tl_gemm_plan(P, P, 0, P, M, N, K, 1, 0, sms, tg.Options(config=config, force_split=int(force)))
        assert s == 0
        if p.tiles_m * p.tiles_n <= 20000:
            if check_schedule(p.as_dict(), sms, K) > 1:
                seen["split"] += 1

    check()
    assert seen["split"] > 50  # the split path was exercised


def test_plan_from_many_threads_matches_one_thread():
    """The planner called from eight threads at once (ctypes releases the GIL
    for each call) returns, for every shape, the plan one thread computes."""
    from concurrent.futures import ThreadPoolExecutor
    rng = np.random.default_rng(5)
    cases = [(int(M), int(N), int(K), int(dt), int(epi))
             for M, N, K, dt, epi in zip(rng.integers(1, 70000, 600), rng.integers(1, 70000, 600),
                                         rng.integers(1, 70000, 600), rng.integers(0, 2, 600),
                                         rng.integers(0, 6, 600))]

    def one(case):
        M, N, K, dt, epi = case
        st, p = tg.tl_gemm_plan(P, P, P if epi in (1, 2, 4) else 0, P, M, N, K, dt, epi, 148, None)
        assert st == 0
        return tuple(sorted(p.as_dict().items()))

    expected = [one(c) for c in cases]
    with ThreadPoolExecutor(max_workers=8) as pool:
        for _ in range(3):
            assert list(pool.map(one, cases)) == expected
