"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics.

Each test would fail under a plausible slip in the oracle: a wrong head
mapping (a % H_kv instead of a / G), a mask off by one or missing the suffix
offset, a missing or wrong scale, a missing normaliser, no max subtraction,
a transposed operand or a wrong row/plane index.
"""
import json
import math
import os

import numpy as np
import pytest

import gqa_inputs as gi
import oracle
from tests.brute_force import brute_force_attention

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# The library the pins run against: None = the committed oracle. The mutation
# test swaps in builds of the oracle with a planted mistake.
LIB = None


def att(*args, **kw):
    return oracle.attention(*args, lib=LIB, **kw)


def att_rows(*args, **kw):
    return oracle.attention_rows(*args, lib=LIB, **kw)


def bits(x):
    """float values that are exact in bf16 -> bf16 bit array (asserts exactness)."""
    x = np.asarray(x, dtype=np.float32)
    b = gi.f32_to_bf16_bits(x).reshape(x.shape)
    assert np.array_equal(gi.bf16_bits_to_f32(b).reshape(x.shape), x), "value not exact in bf16"
    return b


def f64(u16):
    return gi.bf16_bits_to_f32(u16).astype(np.float64).reshape(np.shape(u16))


def rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=0):
    q = gi.normal_bf16(seed, gi.TENSOR_Q, (B, Hq, Tq, D))
    k = gi.normal_bf16(seed, gi.TENSOR_K, (B, Hkv, Tk, D))
    v = gi.normal_bf16(seed, gi.TENSOR_V, (B, Hkv, Tk, D))
    return q, k, v


def test_head_mapping_golden_example():
    """[1,1,7,7]: consecutive query heads share a KV head (the page's own check)."""
    g = json.load(open(os.path.join(GOLDEN, "head_mapping_example.json")))
    q = bits(np.array(g["q"]).reshape(g["q_shape"]))
    k = bits(np.array(g["k"]).reshape(g["k_shape"]))
    v = bits(np.array(g["v"]).reshape(g["k_shape"]))
    out = att(q, k, v)
    assert out.reshape(-1).tolist() == g["expected_flat"]


def test_suffix_consistency_golden_example():
    """Last row of full causal attention == the T_q = 1 suffix call (the page's check)."""
    g = json.load(open(os.path.join(GOLDEN, "suffix_consistency_example.json")))
    B, Hq, Tq, D = g["q_shape"]
    Hkv, Tk = g["kv_shape"][1], g["kv_shape"][2]
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=g["seed"])
    full = att(q, k, v)
    assert full.shape == tuple(g["q_shape"])
    step = att(np.ascontiguousarray(q[:, :, -1:]), k, v)
    np.testing.assert_array_equal(step, full[:, :, -1:])
    # and the same holds for every suffix length, not just 1
    for tq in (2, 3, 4):
        part = att(np.ascontiguousarray(q[:, :, Tq - tq:]), k, v)
        np.testing.assert_array_equal(part, full[:, :, Tq - tq:])


@pytest.mark.parametrize("shape", [
    (2, 4, 2, 5, 5, 8),     # the page's check shapes
    (1, 4, 1, 3, 7, 4),     # MQA, suffix offset 4
    (2, 6, 3, 6, 6, 16),    # G = 2
    (1, 3, 3, 4, 9, 8),     # MHA, suffix offset 5
    (2, 8, 2, 1, 11, 8),    # decode-like T_q = 1
    (1, 2, 1, 17, 17, 32),
])
def test_matches_brute_force_matrix_form(shape):
    B, Hq, Hkv, Tq, Tk, D = shape
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=7)
    ref = brute_force_attention(f64(q), f64(k), f64(v))
    out = att(q, k, v)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_values_all_ones_give_ones():
    """Softmax rows sum to one, so V = 1 gives O = 1."""
    q, k, _ = rand_qkv(2, 4, 2, 9, 13, 16, seed=3)
    v = bits(np.ones(k.shape))
    out = att(q, k, v)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_zero_query_gives_prefix_mean_and_log_count_lse():
    """q = 0 makes every visible score equal: o_i is the mean of v[0..pos], LSE = ln(pos+1)."""
    B, Hq, Hkv, Tq, Tk, D = 1, 4, 2, 5, 12, 8
    _, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=11)
    q = bits(np.zeros((B, Hq, Tq, D)))
    out, lse = att(q, k, v, with_lse=True)
    vf = f64(v)
    for a in range(Hq):
        g = a // (Hq // Hkv)
        for i in range(Tq):
            pos = Tk - Tq + i
            np.testing.assert_allclose(out[0, a, i], vf[0, g, :pos + 1].mean(axis=0), rtol=0, atol=1e-14)
            assert abs(lse[0, a, i] - math.log(pos + 1)) < 1e-14


def test_two_key_closed_form_checks_scale_and_diagonal():
    """One query over two keys with scores 0 and c/sqrt(D): a logistic weight in closed form."""
    D = 4                      # 1/sqrt(4) = 0.5 exactly
    c = 3.0
    q = bits(np.array([c, 0, 0, 0]).reshape(1, 1, 1, D))
    k = bits(np.array([[0, 0, 0, 0], [1, 0, 0, 0]]).reshape(1, 1, 2, D))
    v = bits(np.array([[1, 2, 3, 4], [-5, 6, 0.5, 8]]).reshape(1, 1, 2, D))
    w1 = math.exp(c * 0.5) / (1.0 + math.exp(c * 0.5))
    expect = (1 - w1) * f64(v)[0, 0, 0] + w1 * f64(v)[0, 0, 1]
    out = att(q, k, v)
    np.testing.assert_allclose(out[0, 0, 0], expect, rtol=0, atol=1e-15)
    # With T_q = T_k = 2, query row 0 sits at position 0 and sees only key 0.
    q2 = bits(np.array([[c, 0, 0, 0], [c, 0, 0, 0]]).reshape(1, 1, 2, D))
    out2 = att(q2, k, v)
    np.testing.assert_array_equal(out2[0, 0, 0], f64(v)[0, 0, 0])
    np.testing.assert_allclose(out2[0, 0, 1], expect, rtol=0, atol=1e-15)
    # An explicit scale override replaces 1/sqrt(D).
    out3 = att(q, k, v, scale=1.0)
    w1b = math.exp(c) / (1.0 + math.exp(c))
    np.testing.assert_allclose(out3[0, 0, 0], (1 - w1b) * f64(v)[0, 0, 0] + w1b * f64(v)[0, 0, 1],
                               rtol=0, atol=1e-15)


def test_huge_logits_stay_finite():
    """Scores near 2048 overflow exp() in double unless the row max is subtracted."""
    D = 4
    q = bits(np.array([64, 0, 0, 0]).reshape(1, 1, 1, D))
    k = bits(np.array([[64, 0, 0, 0], [64.5, 0, 0, 0]]).reshape(1, 1, 2, D))  # scores 2048, 2064
    v = bits(np.array([[1, 0, 0, 0], [0, 1, 0, 0]]).reshape(1, 1, 2, D))
    out, lse = att(q, k, v, with_lse=True)
    w1 = 1.0 / (1.0 + math.exp(-16.0))
    np.testing.assert_allclose(out[0, 0, 0], [1 - w1, w1, 0, 0], rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 0] - (2064.0 + math.log1p(math.exp(-16.0)))) < 1e-12


def test_gqa_equals_mha_on_repeated_planes():
    """GQA(K, V) == MHA(repeat_interleave(K, V)) exactly; MQA is the H_kv = 1 case."""
    for Hkv in (1, 2, 4):
        q, k, v = rand_qkv(2, 8, Hkv, 6, 10, 16, seed=5)
        g = 8 // Hkv
        k_rep = np.ascontiguousarray(np.repeat(k, g, axis=1))
        v_rep = np.ascontiguousarray(np.repeat(v, g, axis=1))
        np.testing.assert_array_equal(att(q, k, v), att(q, k_rep, v_rep))


def test_key_permutation_invariance_when_all_keys_visible():
    """With T_q = 1 every key is visible: permuting key/value rows together leaves o unchanged."""
    q, k, v = rand_qkv(1, 4, 2, 1, 23, 16, seed=9)
    perm = np.random.default_rng(0).permutation(23)
    out = att(q, k, v)
    out_p = att(q, np.ascontiguousarray(k[:, :, perm]), np.ascontiguousarray(v[:, :, perm]))
    np.testing.assert_allclose(out_p, out, rtol=0, atol=1e-13)


def test_affine_in_values():
    """o(2V) = 2 o(V) and o(V + c) = o(V) + c, because the weights sum to one."""
    q, k, v = rand_qkv(1, 2, 1, 7, 7, 8, seed=13)
    vf = gi.bf16_bits_to_f32(v).reshape(v.shape)
    out = att(q, k, v)
    out2 = att(q, k, bits(vf * 2))
    np.testing.assert_array_equal(out2, 2 * out)
    vc = np.round(vf * 8) / 8 + 1.0        # values exact in bf16 (|x| < 16 with 3 fraction bits)
    outc = att(q, k, bits(vc))
    outc0 = att(q, k, bits(vc - 1.0))
    np.testing.assert_allclose(outc, outc0 + 1.0, rtol=0, atol=1e-13)


def test_row_subset_matches_full_and_strided_cache():
    B, Hq, Hkv, Tq, Tk, D = 2, 4, 2, 6, 9, 8
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=21)
    full = att(q, k, v).reshape(-1, D)
    rows = np.array([0, 5, 17, 23, B * Hq * Tq - 1])
    np.testing.assert_array_equal(att_rows(q, k, v, rows), full[rows])
    # a cache with capacity 16 whose first Tk positions hold k/v
    cap = 16
    kc = gi.normal_bf16(99, 1, (B, Hkv, cap, D))
    vc = gi.normal_bf16(99, 2, (B, Hkv, cap, D))
    kc[:, :, :Tk] = k
    vc[:, :, :Tk] = v
    np.testing.assert_array_equal(att(q, kc, vc, Tk=Tk).reshape(-1, D), full)


def test_rejects_what_the_pages_assert_against():
    q, k, v = rand_qkv(1, 3, 2, 2, 2, 4)
    with pytest.raises(ValueError):
        att(q, k, v)            # H_q % H_kv != 0
    q, k, v = rand_qkv(1, 2, 1, 5, 4, 4)
    with pytest.raises(ValueError):
        att(q, k, v)            # T_q > T_k


def test_threads_do_not_change_results():
    q, k, v = rand_qkv(2, 4, 2, 33, 40, 16, seed=4)
    np.testing.assert_array_equal(att(q, k, v, threads=1), att(q, k, v, threads=8))


# ---------------------------------------------------------------- sliding window
def test_window_of_one_returns_the_own_value_row():
    """w = 1: each query sees only its own position, so o = v[pos] and LSE = its own score."""
    B, Hq, Hkv, Tq, Tk, D = 1, 4, 2, 6, 9, 8
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=31)
    out, lse = att(q, k, v, window=1, with_lse=True)
    qf, kf, vf = f64(q), f64(k), f64(v)
    for a in range(Hq):
        g = a // (Hq // Hkv)
        for i in range(Tq):
            pos = Tk - Tq + i
            np.testing.assert_array_equal(out[0, a, i], vf[0, g, pos])
            assert abs(lse[0, a, i] - qf[0, a, i] @ kf[0, g, pos] / math.sqrt(D)) < 1e-12


def test_window_zero_query_gives_window_mean():
    """q = 0 inside a window of w: o_i is the mean of v over positions max(0, pos-w+1)..pos."""
    B, Hq, Hkv, Tq, Tk, D, w = 1, 2, 1, 7, 13, 8, 4
    _, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=33)
    q = bits(np.zeros((B, Hq, Tq, D)))
    out, lse = att(q, k, v, window=w, with_lse=True)
    vf = f64(v)
    for i in range(Tq):
        pos = Tk - Tq + i
        lo = max(0, pos - w + 1)
        np.testing.assert_allclose(out[0, 0, i], vf[0, 0, lo:pos + 1].mean(axis=0), rtol=0, atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(pos + 1 - lo)) < 1e-14


@pytest.mark.parametrize("shape,w", [((2, 4, 2, 9, 9, 8), 3), ((1, 4, 1, 5, 12, 4), 5), ((1, 3, 3, 8, 8, 16), 1),
                                     ((2, 2, 1, 1, 10, 8), 4)])
def test_window_matches_brute_force_matrix_form(shape, w):
    B, Hq, Hkv, Tq, Tk, D = shape
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=35)
    ref = brute_force_attention(f64(q), f64(k), f64(v), window=w)
    np.testing.assert_allclose(att(q, k, v, window=w), ref, rtol=0, atol=1e-12)


def test_window_at_least_the_context_is_plain_causal():
    q, k, v = rand_qkv(1, 4, 2, 6, 10, 8, seed=37)
    full = att(q, k, v)
    for w in (10, 11, 1000):
        np.testing.assert_array_equal(att(q, k, v, window=w), full)
    assert not np.array_equal(att(q, k, v, window=9), full)


def test_window_suffix_consistency():
    """The pages' suffix check also holds under a window."""
    q, k, v = rand_qkv(2, 4, 2, 6, 6, 8, seed=39)
    full = att(q, k, v, window=3)
    np.testing.assert_array_equal(att(np.ascontiguousarray(q[:, :, -2:]), k, v, window=3), full[:, :, -2:])
