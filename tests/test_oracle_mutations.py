"""The oracle pins catch plausible mistakes.

Each case compiles a copy of the oracle source with one planted mistake (on the
CPU, in a temporary directory) and runs the pin tests against it: at least one
pin must fail.  This shows the pins constrain every term of the definition
(scale, V columns, causal offset, kv-head mapping, page indexing, LSE base, the
combine weights, the FP8 cache's scale blocks, e4m3 exponent bias and
subnormals, RoPE offset and bfloat16 rounding, the sparse decode's scale, LSE
and V columns, and the sparse prefill's log2(e), LSE base, weights and V columns).
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import tests.test_oracle_fp8_pins as fp8_pins
import tests.test_oracle_prefill_pins as prefill_pins
import tests.test_oracle_sparse_pins as sparse_pins
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "mla_oracle.c")

MUTATIONS = {
    "causal_offset": ("L - sh->s_q + 1 + s", "L - sh->s_q + s"),
    "dropped_scale": ("x[j - lo] = sh->scale * acc;", "x[j - lo] = acc;"),
    "v_wrong_columns": ("o_row[d] += w * mla_oracle_half_to_double(vp[d], sh->dtype)",
                        "o_row[d] += w * mla_oracle_half_to_double(vp[d + sh->d_qk - sh->dv], sh->dtype)"),
    "lse_base2": ("double lse = M + log(sum);", "double lse = M + log2(sum);"),
    "kv_head_map": ("const int g = h / (sh->h_q / sh->h_kv);", "const int g = h % sh->h_kv;"),
    "page_offset": ("(((size_t)page * P + (j % P))", "(((size_t)page * P + (j / P))"),
    "combine_weight": ("double w = exp(lse_parts[(size_t)k * rows + r] - L);",
                       "double w = exp(lse_parts[(size_t)k * rows + r] - M);"),
    # the "FP8 with scale" cache
    "fp8_scale_block": ("* (double)scale[i / 128];", "* (double)scale[(i / 64) % 4];"),
    "fp8_exponent_bias": ("e - 10); /* (1 + m / 8)", "e - 11); /* (1 + m / 8)"),
    "fp8_subnormal": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "fp8_rope_offset": ("row + 528 + 2 * i", "row + 526 + 2 * i"),
    "bf16_truncation": ("if (rest > 0x8000u || (rest == 0x8000u && (hi & 1u))) hi += 1;", ""),
    "bf16_ties_away": ("(rest == 0x8000u && (hi & 1u))", "(rest == 0x8000u)"),
    # token-level sparse decoding
    "sparse_dropped_scale": ("x[k] = sh->scale * acc;", "x[k] = acc;"),
    "sparse_lse_without_sum": ("const double L = M + log(sum);", "const double L = M;"),
    "sparse_v_wrong_columns": ("o_row[d] += w * mla_oracle_half_to_double(vp[d], sh->dtype);\n                }\n            }\n        }",
                               "o_row[d] += w * mla_oracle_half_to_double(vp[d + d_qk - dv], sh->dtype);\n                }\n            }\n        }"),
    # the sparse prefill
    "prefill_dropped_log2e": ("P[k] = acc * sm_scale * log2e;", "P[k] = acc * sm_scale;"),
    "prefill_lse_natural_log": ("const double l2 = mx + log2(sum);", "const double l2 = mx + log(sum);"),
    "prefill_weights_unnormalized": ("const double w = exp2(P[k] - l2);", "const double w = exp2(P[k] - mx);"),
    "prefill_v_wrong_columns": ("o_row[d] += w * mla_oracle_half_to_double(vp[d], dtype);",
                                "o_row[d] += w * mla_oracle_half_to_double(vp[d + d_qk - dv], dtype);"),
    "prefill_kv_head_map": ("const int32_t* ix = indices + ((size_t)i * h_kv + g) * topk;",
                            "const int32_t* ix = indices + ((size_t)i * h_kv) * topk;"),
}


def _pin_calls():
    """(name, zero-arg callable) for every pin that takes only the oracle module."""
    calls = []
    for case in pins._parse_golden():
        calls.append((f"hand:{case['name']}", lambda c=case: pins.test_hand_cases(oracle, c)))
    for kw in pins.BRUTE_CASES:
        calls.append((f"brute:{kw['seqlens']}", lambda k=kw: pins.test_brute_force_torch(oracle, k)))
    for name in ("test_single_visible_token", "test_zero_query_is_mean_of_values",
                 "test_identical_keys_give_uniform_weights", "test_empty_sequence",
                 "test_lse_is_logsumexp_of_scaled_logits", "test_weights_sum_to_one"):
        calls.append((name, lambda f=getattr(pins, name): f(oracle)))
    for causal in (False, True):
        calls.append((f"split_combine:{causal}",
                      lambda c=causal: pins.test_split_then_combine_equals_unsplit(oracle, c)))
    for name in ("test_e4m3_all_codes_match_torch", "test_dequant_hand_row",
                 "test_dequant_random_rows_match_torch"):
        calls.append((name, lambda f=getattr(fp8_pins, name): f(oracle)))
    for args in [(0x3A, 0.828125, 0x3F84), (0x3D, 1.2109375, 0x3FFC), (0x3C, 1.0078125, 0x3FC2)]:
        calls.append((f"fp8_rounding:{args}",
                      lambda a=args: fp8_pins.test_dequant_rounds_to_nearest_even(oracle, *a)))
    for kw in sparse_pins.SPARSE_CASES:
        calls.append((f"sparse_brute:{kw['seqlens']}",
                      lambda k=kw: sparse_pins.test_sparse_brute_force_torch(oracle, k)))
    for name in ("test_one_row_listed_n_times", "test_full_token_list_equals_dense_decode"):
        calls.append((name, lambda f=getattr(sparse_pins, name): f(oracle)))
    for kw in prefill_pins.PREFILL_CASES:
        calls.append((f"prefill_brute:{kw}", lambda k=kw: prefill_pins.test_prefill_brute_force_torch(oracle, k)))
    for name in ("test_prefill_hand_two_entries", "test_prefill_single_entry_and_no_entry",
                 "test_prefill_row_listed_n_times", "test_prefill_is_the_sparse_decode_in_base_2"):
        calls.append((name, lambda f=getattr(prefill_pins, name): f(oracle)))
    for kw in fp8_pins.FP8_BRUTE_CASES:
        calls.append((f"fp8_brute:{kw['seqlens']}",
                      lambda k=kw: fp8_pins.test_fp8_decode_brute_force_torch(oracle, k)))
    return calls


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert old in src, f"mutation anchor for {name} not found in the oracle source"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o",
                           str(lib), str(mutant), "-lm"])
    failed = []
    with oracle.use_library(str(lib)):
        for pin_name, call in _pin_calls():
            try:
                call()
            except (AssertionError, ValueError):
                failed.append(pin_name)
    assert failed, f"no pin caught the planted mistake {name!r}"


def test_unmutated_source_passes_every_pin():
    with oracle.use_library(oracle.build()):
        for _, call in _pin_calls():
            call()
