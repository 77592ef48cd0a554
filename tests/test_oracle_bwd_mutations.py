"""The backward pins have teeth: plant plausible mistakes in copies of the oracle's
backward (CPU only), build each copy and check that at least one pin fails."""
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_bwd_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gqa_oracle.c")

# (name, text, replacement, which occurrence to replace: -1 = the last)
MUTATIONS = [
    ("row term of the softmax Jacobian dropped", "const double ds = p[j] * (dp[j] - rowterm);",
     "const double ds = p[j] * dp[j];", -1),
    ("value gradient with unnormalised weights", "for (long long j = first; j <= pos; ++j) p[j] /= l;",
     "(void)l;", -1),
    ("key gradient without the scale", "dk[j * D + d] += J->scale * ds * qd[d];",
     "dk[j * D + d] += ds * qd[d];", -1),
    ("query gradient from the values", "dqrow[d] += J->scale * ds * bf16_to_double(kplane[j * D + d]);",
     "dqrow[d] += J->scale * ds * bf16_to_double(vplane[j * D + d]);", -1),
    ("group sum dropped", "for (long long a = g * group; a < (g + 1) * group; ++a) {",
     "for (long long a = g * group; a < g * group + 1; ++a) {", -1),
    ("value gradient from the queries", "dv[j * D + d] += p[j] * dod[d];", "dv[j * D + d] += p[j] * qd[d];", -1),
    ("window ignored in the backward",
     "const long long first = (J->window > 0 && pos - J->window + 1 > 0) ? pos - J->window + 1 : 0;",
     "const long long first = 0;", -1),
]

PIN_TESTS = [(pins.test_gradients_match_finite_differences_of_the_matrix_form, {"case": c})
             for c in pins.FD_CASES] + [
    (pins.test_key_gradient_columns_sum_to_zero, {}),
    (pins.test_uniform_weights_give_the_value_gradient_in_closed_form, {}),
    (pins.test_gqa_gradients_are_mha_gradients_summed_over_the_group, {}),
]


@pytest.mark.parametrize("name,old,new,which", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new, which, tmp_path):
    src = open(SRC).read()
    assert old in src, f"mutation anchor not found: {old!r}"
    at = src.rfind(old) if which == -1 else src.find(old)
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src[:at] + new + src[at + len(old):])
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
