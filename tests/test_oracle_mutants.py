"""Plants plausible mistakes in copies of the CPU oracle and checks that the pins
catch each one (no GPU).  The oracle source itself is untouched: every mutant is
a text substitution into a temporary copy, compiled into a temporary library."""
import os

import pytest

import oracle
from tests import oracle_pins as P

MUTANTS = [
    ("k_divisor_128", "quantize_group(x + i * D, D, 127.0f, -127, 127, tmp)",
     "quantize_group(x + i * D, D, 128.0f, -127, 127, tmp)"),
    ("scale_not_rounded_to_f16", "float s = f16_bits_to_f32(sb);", "float s = s32;"),
    ("round_half_up", "static float rne(float x) { return nearbyintf(x); }",
     "static float rne(float x) { return floorf(x + 0.5f); }"),
    ("round_half_away", "static float rne(float x) { return nearbyintf(x); }",
     "static float rne(float x) { return roundf(x); }"),
    ("truncate", "static float rne(float x) { return nearbyintf(x); }",
     "static float rne(float x) { return truncf(x); }"),
    ("reciprocal_multiply", "float r = rne(x[c] / s);", "float r = rne(x[c] * (1.0f / s));"),
    ("nibbles_swapped", "(uint8_t)(lo | (hi << 4))", "(uint8_t)(hi | (lo << 4))"),
    ("v_clamp_symmetric", "quantize_group(x + i * D + g * 32, 32, 7.0f, -8, 7, codes)",
     "quantize_group(x + i * D + g * 32, 32, 7.0f, -7, 7, codes)"),
    ("v_divisor_8", "quantize_group(x + i * D + g * 32, 32, 7.0f, -8, 7, codes)",
     "quantize_group(x + i * D + g * 32, 32, 8.0f, -8, 7, codes)"),
    ("v_group_16", "scales[i * G + g] = quantize_group(x + i * D + g * 32, 32,",
     "scales[i * G + g] = quantize_group(x + i * D + g * 32, 16,"),
    ("nibble_sign", "return (n & 0x8u) ? (int)n - 16 : (int)n;", "return (n & 0x8u) ? (int)n - 8 : (int)n;"),
    ("gqa_modulo", "const int j = r / Hq, h = r % Hq, hk = h / G;\n        const int64_t n_vis = L - n_q + j + 1;   /* visible",
     "const int j = r / Hq, h = r % Hq, hk = h % Hkv;\n        const int64_t n_vis = L - n_q + j + 1;   /* visible"),
    ("causal_off_by_one", "const int64_t n_vis = L - n_q + j + 1;   /* visible", "const int64_t n_vis = L - n_q + j;   /* visible"),
    ("no_scale", "z[t] = scale * dot;\n            if (z[t] > m) m = z[t];\n        }\n        double l = 0.0;\n        for (int64_t t = 0; t < n_vis; t++) { z[t] = exp(z[t] - m); l += z[t]; }\n        double* o = out + (int64_t)r * D;\n        for (int c = 0; c < D; c++) o[c] = 0.0;\n        for (int64_t t = 0; t < n_vis; t++) {\n            const double w = z[t] / l;\n            const double* vt",
     "z[t] = dot;\n            if (z[t] > m) m = z[t];\n        }\n        double l = 0.0;\n        for (int64_t t = 0; t < n_vis; t++) { z[t] = exp(z[t] - m); l += z[t]; }\n        double* o = out + (int64_t)r * D;\n        for (int c = 0; c < D; c++) o[c] = 0.0;\n        for (int64_t t = 0; t < n_vis; t++) {\n            const double w = z[t] / l;\n            const double* vt"),
    ("unnormalised", "const double w = z[t] / l;\n            const double* vt", "const double w = z[t];\n            const double* vt"),
    ("lse_without_max", "lse[r] = m + log(l);\n        free(z);\n    }\n}\n\n/* Same attention",
     "lse[r] = log(l);\n        free(z);\n    }\n}\n\n/* Same attention"),
    ("absmax_signed", "float m = fabsf(x[c]);", "float m = x[c];"),
    ("draft_earliest_match", "for (int32_t i = L - n - 1; i >= 0; i--) {", "for (int32_t i = 0; i < L - n; i++) {"),
    ("draft_suffix_matches_itself", "for (int32_t i = L - n - 1; i >= 0; i--) {", "for (int32_t i = L - n; i >= 0; i--) {"),
    ("draft_count_off_by_one", "int32_t cnt = L - i - n;", "int32_t cnt = L - i - n - 1;"),
    ("draft_last_token_only", "for (int32_t j = 0; j < n && same; j++) same = tokens[i + j] == tokens[L - n + j];",
     "same = tokens[i + n - 1] == tokens[L - 1];"),
]


def _checks():
    # the cheap, sharp checks first; a mutant stops at its first failure
    order = [P.check_k_hand, P.check_v_hand, P.check_dequant_hand, P.check_memory_claim,
             P.check_attn_single_token, P.check_attn_two_token_closed_form, P.check_attn_weights,
             P.check_attn_gqa, P.check_attn_causal, P.check_attn_torch, P.check_attn_quant_form,
             P.check_roundtrip, P.check_tiny_scales, P.check_near_ties, P.check_k_bruteforce, P.check_v_bruteforce,
             P.check_draft_hand, P.check_draft_rfind]
    return order


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "mq_oracle.c")).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mpath = tmp_path / "mq_oracle_mutant.c"
    mpath.write_text(src.replace(old, new))
    lib = oracle.OracleLib(oracle.build(force=True, src=str(mpath), out=str(tmp_path / "libmutant.so")))
    caught = None
    for check in _checks():
        try:
            check(lib)
        except (AssertionError, ValueError, IndexError, ZeroDivisionError, OverflowError) as e:
            caught = (check.__name__, type(e).__name__)
            break
    assert caught is not None, f"mutant {name} passed every pin"
