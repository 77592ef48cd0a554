"""The shared input generator: deterministic, index-addressable, N(0,1), bf16 RNE."""
import numpy as np

import gqa_inputs as gi


def test_deterministic_and_index_addressable():
    a = gi.normal_bf16(0, 1, (4, 1000), threads=1)
    b = gi.normal_bf16(0, 1, (4, 1000), threads=8)
    np.testing.assert_array_equal(a, b)
    flat = a.reshape(-1)
    for start in (0, 1, 7, 998, 2001):
        part = gi.normal_bf16(0, 1, (333,), start=start)
        np.testing.assert_array_equal(part, flat[start:start + 333])


def test_streams_differ_by_seed_and_tensor():
    a = gi.normal_bf16(0, 0, (4096,))
    assert not np.array_equal(a, gi.normal_bf16(0, 1, (4096,)))
    assert not np.array_equal(a, gi.normal_bf16(1, 0, (4096,)))


def test_standard_normal_moments():
    x = gi.bf16_bits_to_f32(gi.normal_bf16(0, 2, (1 << 20,))).astype(np.float64)
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1.0) < 5e-3
    assert abs((np.abs(x) < 1).mean() - 0.6827) < 3e-3


def test_bf16_round_to_nearest_even():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9], dtype=np.float32)
    b = gi.f32_to_bf16_bits(f)
    back = gi.bf16_bits_to_f32(b)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1); 1 + 3*2^-8 -> 1 + 2^-6 (even)
    np.testing.assert_array_equal(back, np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0], dtype=np.float32))


def test_pow2_scaling_is_exact():
    q = gi.normal_bf16(0, 0, (1000,))
    q4 = gi.scale_pow2_bf16(q, 2)
    np.testing.assert_array_equal(gi.bf16_bits_to_f32(q4), gi.bf16_bits_to_f32(q) * 4)


def test_workload_shapes():
    w = gi.WORKLOADS["mha_suffix"]
    assert w.q_shape == (8, 16, 512, 128) and w.kv_shape == (8, 16, 8192, 128) and w.q_pow2 == 2
    assert gi.WORKLOADS["gqa_decode"].Tq == 1
    t = gi.TINY
    q, k, v = t.make(threads=2)
    assert q.shape == (2, 4, 128, 64) and k.shape == (2, 2, 128, 64) and v.dtype == np.uint16


def test_integer_draws_are_seeded_and_in_range():
    a = gi.uniform_ints(0, gi.STREAM_LEN, 1000, 256, 8192)
    np.testing.assert_array_equal(a, gi.uniform_ints(0, gi.STREAM_LEN, 1000, 256, 8192))
    assert a.min() >= 256 and a.max() <= 8192 and len(set(a.tolist())) > 900
    assert not np.array_equal(a, gi.uniform_ints(1, gi.STREAM_LEN, 1000, 256, 8192))
    p = gi.permutation(0, gi.STREAM_PAGES, 777)
    np.testing.assert_array_equal(np.sort(p), np.arange(777))
    w = gi.words(3, 4, 10)
    np.testing.assert_array_equal(w[4:], gi.words(3, 4, 6, start=4))


def test_varlen_and_paged_workload_recipes():
    w = gi.WORKLOADS.get("tiny")
    assert w is not None
    vw = gi.VARLEN_WORKLOADS["chunked_prefill"]
    lq, lk = vw.lengths()
    assert (lq >= vw.q_lo).all() and (lq <= vw.q_hi).all() and (lk >= lq).all()
    pw = gi.PagedDecodeWorkload("t", 3, 4, 2, 8, 5, 40, 16)
    q, k, v, lens, table = pw.make()
    n_pages = (lens + 15) // 16
    assert k.shape == (int(n_pages.sum()), 16, 2, 8) and q.shape == (3, 4, 1, 8)
    used = np.sort(np.concatenate([table[b, :n_pages[b]] for b in range(3)]))
    np.testing.assert_array_equal(used, np.arange(int(n_pages.sum())))   # every page once
    assert all((table[b, n_pages[b]:] == -1).all() for b in range(3))
