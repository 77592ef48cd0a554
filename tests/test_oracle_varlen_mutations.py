"""The variable-length pins have teeth: plant plausible mistakes in copies of
``oracle/varlen.py`` (CPU only), load each copy as a module of the oracle package and
check that at least one pin fails. The committed file is never modified.
"""
import importlib.util
import os

import pytest

import oracle.varlen
import tests.test_oracle_varlen_pins as pins

SRC = oracle.varlen.__file__

MUTATIONS = [
    ("padded lengths ignored", "length = rows if lens is None else int(lens[s])", "length = rows"),
    ("keys cut to the query length (cached prefix dropped)",
     "ks = _plane(k, b_k, r_k, l_k, packed_k)\n        vs = _plane(v, b_k, r_k, l_k, packed_k)",
     "ks = _plane(k, b_k, r_k, l_q, packed_k)\n        vs = _plane(v, b_k, r_k, l_q, packed_k)"),
    ("keys start at the query's first row",
     "ks = _plane(k, b_k, r_k, l_k, packed_k)\n        vs = _plane(v, b_k, r_k, l_k, packed_k)",
     "ks = _plane(k, b_k, r_q, l_k, packed_k)\n        vs = _plane(v, b_k, r_q, l_k, packed_k)"),
    ("window dropped", "with_lse=with_lse,\n                               window=window)",
     "with_lse=with_lse,\n                               window=0)"),
    ("output rows misplaced", "out[:, r_q:r_q + l_q] = o_s", "out[:, r_k:r_k + l_q] = o_s"),
    ("page table ignored", "pool[table[b, t // page], :, t % page]", "pool[t // page, :, t % page]"),
    ("page row and page swapped", "pool[table[b, t // page], :, t % page]",
     "pool[table[b, t % page], :, t // page]"),
]

PIN_TESTS = [
    (pins.test_packed_matches_segment_mask_matrix_form, {"case": c}) for c in pins.PACKED_CASES
] + [
    (pins.test_padded_ignores_padding_and_matches_segment_mask, {}),
    (pins.test_packed_queries_over_a_padded_cache, {}),
    (pins.test_equal_lengths_packed_equals_dense_batch, {}),
    (pins.test_gather_pages_matches_an_element_loop, {}),
    (pins.test_paged_cache_decode_equals_contiguous_cache, {}),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new, tmp_path):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    path = tmp_path / "varlen_mutant.py"
    path.write_text(src.replace(old, new), encoding="utf-8")
    spec = importlib.util.spec_from_file_location("oracle._varlen_mutant", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    caught = []
    saved = pins.OV
    pins.OV = mod
    try:
        for fn, kw in PIN_TESTS:
            try:
                fn(**kw)
            except (AssertionError, ValueError, IndexError):
                caught.append(fn.__name__)
    finally:
        pins.OV = saved
    assert caught, f"no pin caught the planted mistake: {name}"
