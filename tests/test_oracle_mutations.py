"""The pins have teeth: plant plausible mistakes in copies of the oracle's C
source (CPU only), build each copy, and check that at least one pin fails.

The committed oracle itself is never modified; each mutant is a temporary
file compiled into a temporary library.
"""
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gqa_oracle.c")

# (name, text in the oracle, replacement): each is a mistake a careful reader
# could make when writing the definition out.
MUTATIONS = [
    ("head mapping a % H_kv", "const long long g = a / group;", "const long long g = a % J->Hkv;"),
    ("diagonal excluded", "j <= pos", "j < pos"),
    ("suffix offset dropped", "(long long)(J->Tk - J->Tq) + i;", "i;"),
    ("scale dropped", "s[j] = J->scale * acc;", "s[j] = acc;"),
    ("scale 1/D instead of 1/sqrt(D)", "1.0 / sqrt((double)D)", "1.0 / (double)D"),
    ("normaliser dropped", "for (int d = 0; d < D; ++d) o[d] /= l;", "(void)l;"),
    ("no max subtraction", "s[j] = exp(s[j] - m);", "s[j] = exp(s[j]);"),
    ("keys used as values", "J->v + b * J->v_sb + g * J->v_sh", "J->k + b * J->k_sb + g * J->k_sh"),
    ("query row index dropped", "a * J->q_sh + i * D;", "a * J->q_sh;"),
    ("batch stride of K dropped", "J->k + b * J->k_sb + g * J->k_sh", "J->k + g * J->k_sh"),
    ("LSE without log", "*lse_out = m + log(l);", "*lse_out = m + l;"),
    ("query and key swapped in the group", "a / group;", "a / J->Hkv;"),
    ("window one key too wide", "pos - J->window + 1 > 0) ? pos - J->window + 1 : 0;",
     "pos - J->window > 0) ? pos - J->window : 0;"),
    ("window one key too narrow", "pos - J->window + 1 > 0) ? pos - J->window + 1 : 0;",
     "pos - J->window + 2 > 0) ? pos - J->window + 2 : 0;"),
    ("window ignored", "(J->window > 0 && pos", "(0 && pos"),
]

PIN_TESTS = [
    (pins.test_head_mapping_golden_example, {}),
    (pins.test_suffix_consistency_golden_example, {}),
    (pins.test_matches_brute_force_matrix_form, {"shape": (2, 4, 2, 5, 5, 8)}),
    (pins.test_matches_brute_force_matrix_form, {"shape": (1, 4, 1, 3, 7, 4)}),
    (pins.test_values_all_ones_give_ones, {}),
    (pins.test_zero_query_gives_prefix_mean_and_log_count_lse, {}),
    (pins.test_two_key_closed_form_checks_scale_and_diagonal, {}),
    (pins.test_huge_logits_stay_finite, {}),
    (pins.test_gqa_equals_mha_on_repeated_planes, {}),
    (pins.test_affine_in_values, {}),
    (pins.test_row_subset_matches_full_and_strided_cache, {}),
    (pins.test_window_of_one_returns_the_own_value_row, {}),
    (pins.test_window_zero_query_gives_window_mean, {}),
    (pins.test_window_matches_brute_force_matrix_form, {"shape": (2, 4, 2, 9, 9, 8), "w": 3}),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new, tmp_path):
    src = open(SRC).read()
    assert old in src, f"mutation anchor not found: {old!r}"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib_path = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", str(lib_path), str(mutant),
                           "-lm", "-lpthread"])
    lib = oracle.load_variant(str(lib_path))
    caught = []
    saved = pins.LIB
    pins.LIB = lib
    try:
        for fn, kw in PIN_TESTS:
            try:
                fn(**kw)
            except (AssertionError, ValueError, FloatingPointError):
                caught.append(fn.__name__)
    finally:
        pins.LIB = saved
    assert caught, f"no pin caught the planted mistake: {name}"
