"""Plant plausible mistakes in copies of the oracle (on the CPU) and show that
each one fails at least one pin.  The copies are built in a temporary folder;
the oracle in oracle/ is never modified."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
from oracle_pins import ALL_PINS  # noqa: E402
from oracle_pins_attention import ATTENTION_PINS  # noqa: E402
from oracle_pins_elementwise import ELEMENTWISE_PINS  # noqa: E402

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, text in oracle.c, replacement).  Every replacement stays in bounds.
MUTANTS = [
    ("transposed_B_rows", "c[j] += a * b[j];", "c[j] += a * Bd[j * K + k];"),
    ("transposed_B_points", "decode(B[k * N + j], dtype)", "decode(B[j * K + k], dtype)"),
    ("dropped_first_k", "for (int64_t k = 0; k < K; ++k) {", "for (int64_t k = 1; k < K; ++k) {"),
    ("wrong_sign", "c[j] += a * b[j];", "c[j] -= a * b[j];"),
    ("float_accumulator", "c[j] += a * b[j];", "c[j] = (float)(c[j] + a * b[j]);"),
    ("tanh_gelu", "return 0.5 * x * erfc(-x / sqrt(2.0));",
     "return 0.5 * x * (1.0 + tanh(0.7978845608028654 * (x + 0.044715 * x * x * x)));"),
    ("gelu_wrong_scale", "erfc(-x / sqrt(2.0))", "erfc(-x / 2.0)"),
    ("gelu_cancelling_form", "return 0.5 * x * erfc(-x / sqrt(2.0));",
     "return 0.5 * x * (1.0 + erf(x / sqrt(2.0)));"),
    ("gelu_wrong_sign_in_erfc", "erfc(-x / sqrt(2.0))", "erfc(x / sqrt(2.0))"),
    ("bias_after_gelu",
     "    if (epi_has_bias(epi))\n        s = s + decode(bias[j], dtype);\n"
     "    if (epi == ORACLE_EPI_BIAS_GELU || epi == ORACLE_EPI_GELU)\n        s = oracle_gelu(s);",
     "    if (epi == ORACLE_EPI_BIAS_GELU || epi == ORACLE_EPI_GELU)\n        s = oracle_gelu(s);\n"
     "    if (epi_has_bias(epi))\n        s = s + decode(bias[j], dtype);"),
    ("bias_by_row", "c[j] = epilogue(c[j], bias, j, dtype, epi);", "c[j] = epilogue(c[j], bias, i % N, dtype, epi);"),
    ("bias_only_drops_bias", "return epi == ORACLE_EPI_BIAS_GELU || epi == ORACLE_EPI_BIAS || ",
     "return epi == ORACLE_EPI_BIAS_GELU || "),
    ("gelu_only_adds_bias", "        s = oracle_gelu(s);", "        s = oracle_gelu(epi == ORACLE_EPI_GELU ? s + 1.0 : s);"),
    ("gelu_only_skips_gelu", "if (epi == ORACLE_EPI_BIAS_GELU || epi == ORACLE_EPI_GELU)", "if (epi == ORACLE_EPI_BIAS_GELU)"),
    ("tanh_epilogue_uses_erf", "s = oracle_gelu_tanh(s);", "s = oracle_gelu(s);"),
    ("tanh_without_cubic", "(x + 0.044715 * x * x * x)", "(x)"),
    ("tanh_wrong_cubic_coefficient", "0.044715 * x * x * x", "0.04715 * x * x * x"),
    ("tanh_wrong_scale", "sqrt(2.0 / M_PI)", "sqrt(1.0 / M_PI)"),
    ("tanh_cancelling_form", "return u >= 0.0 ? x / (1.0 + e) : x * e / (1.0 + e);",
     "return 0.5 * x * (1.0 + tanh(u));"),
    ("tanh_overflowing_form", "return u >= 0.0 ? x / (1.0 + e) : x * e / (1.0 + e);",
     "return x / (1.0 + exp(-2.0 * u));"),
    ("tanh_branches_swapped", "return u >= 0.0 ? x / (1.0 + e)", "return u < 0.0 ? x / (1.0 + e)"),
    ("tanh_bias_dropped", " || epi == ORACLE_EPI_BIAS_GELU_TANH;", ";"),
    ("tanh_only_skips_gelu", "else if (epi == ORACLE_EPI_BIAS_GELU_TANH || epi == ORACLE_EPI_GELU_TANH)",
     "else if (epi == ORACLE_EPI_BIAS_GELU_TANH)"),
    ("attn_mask_wrong_direction", "const int64_t nkeys = causal ? (i + 1 < Sk ? i + 1 : Sk) : Sk;",
     "const int64_t nkeys = causal ? (i < Sk ? i : Sk) + (i == 0) : Sk;"),
    ("attn_scale_ignored", "s[j] = scale * acc;", "s[j] = acc;"),
    ("attn_scale_squared", "s[j] = scale * acc;", "s[j] = scale * scale * acc;"),
    ("attn_mask_bottom_right", "const int64_t nkeys = causal ? (i + 1 < Sk ? i + 1 : Sk) : Sk;",
     "const int64_t off = Sk > Sq ? Sk - Sq : 0;\n"
     "        const int64_t nkeys = causal ? (i + 1 + off < Sk ? i + 1 + off : Sk) : Sk;"),
    ("attn_k_from_next_head", "const uint16_t *k = K + (bh * Sk + j) * D;",
     "const uint16_t *k = K + (((bh + 1) % BH) * Sk + j) * D;"),
    ("attn_no_max_subtraction", "const double w = exp(s[j] - m);", "const double w = exp(s[j]);"),
    ("attn_unnormalised", "o[d] /= l;", "o[d] /= 1.0;"),
    ("attn_v_from_query_row", "const uint16_t *v = V + (bh * Sk + j) * D;",
     "const uint16_t *v = V + (bh * Sk + (j + i) % Sk) * D;"),
    ("attn_lse_without_max", "lse[p] = m + log(l);", "lse[p] = log(l);"),
    ("softmax_no_max_subtraction", "            y[j] = exp(y[j] - m);", "            y[j] = exp(y[j]);"),
    ("softmax_unnormalised", "            y[j] /= s;", "            y[j] /= 1.0;"),
    ("softmax_max_of_first_only", "            if (y[j] > m)\n                m = y[j];",
     "            if (j == 0)\n                m = y[j];"),
    ("vector_add_in_float_twice", "C[i] = (float)((double)A[i] + (double)B[i]);",
     "C[i] = (float)((double)A[i] + (double)(float)(B[i] * 1.0000001f));"),
    ("f16_exponent_bias", "v = ldexp((double)(f + 1024), e - 25);", "v = ldexp((double)(f + 1024), e - 24);"),
    ("f16_subnormal_as_normal", "v = ldexp((double)f, -24);", "v = ldexp((double)(f + 1024), -25);"),
    ("bf16_exponent_bias", "v = ldexp((double)(f + 128), e - 134);", "v = ldexp((double)(f + 128), e - 133);"),
    ("bf16_fraction_width", "int f = h & 0x7f;", "int f = h & 0x3f;"),
    ("last_k_dropped_points", "for (int64_t k = 0; k < K; ++k)\n            s +=",
     "for (int64_t k = 0; k + 1 < K; ++k)\n            s +="),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_fails_a_pin(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    csrc = tmp_path / f"oracle_{name}.c"
    csrc.write_text(mutated)
    so = oracle.build(force=True, src=str(csrc), out=str(tmp_path / f"liboracle_{name}.so"))
    orc = oracle.from_library(so)
    failed = []
    for pin in ALL_PINS + ATTENTION_PINS + ELEMENTWISE_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
            break
    assert failed, f"mutant {name} passed every pin"
