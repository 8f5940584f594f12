"""The oracle pins catch plausible mistakes.

Each case compiles a copy of the oracle source with one planted mistake (on the
CPU, in a temporary directory) and runs the pin tests against it: at least one
pin must fail.  This shows the pins constrain every term of the definition
(scale, V columns, causal offset, kv-head mapping, page indexing, LSE base, the
combine weights).
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "mla_oracle.c")

MUTATIONS = {
    "causal_offset": ("L - sh->s_q + 1 + s", "L - sh->s_q + s"),
    "dropped_scale": ("x[j - lo] = sh->scale * acc;", "x[j - lo] = acc;"),
    "v_wrong_columns": ("o_row[d] += w * mla_oracle_half_to_double(vp[d]",
                        "o_row[d] += w * mla_oracle_half_to_double(vp[d + sh->d_qk - sh->dv]"),
    "lse_base2": ("double lse = M + log(sum);", "double lse = M + log2(sum);"),
    "kv_head_map": ("const int g = h / (sh->h_q / sh->h_kv);", "const int g = h % sh->h_kv;"),
    "page_offset": ("(((size_t)page * P + (j % P))", "(((size_t)page * P + (j / P))"),
    "combine_weight": ("double w = exp(lse_parts[(size_t)k * rows + r] - L);",
                       "double w = exp(lse_parts[(size_t)k * rows + r] - M);"),
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
