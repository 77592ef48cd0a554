"""Pins for the variable-length, padded and paged forms of the oracle (CPU only).

The oracle slices every sequence out and calls the dense row oracle on it. The main
pin is a different formulation: one score matrix over the whole flattened token
axis, per head, with an explicit segment mask built here from the sequence bounds
("注意力家族", section Mask 与增量位置: padding / packed segment masks, and masks
built from absolute positions, not from the tensors' shapes). A slip in the
oracle's slicing (a wrong start row, the query length used for the keys, a dropped
cached prefix, a misplaced output row) changes which keys a row sees and fails it.
"""
import numpy as np
import pytest

import gqa_inputs as gi
import oracle.varlen
from tests.brute_force import brute_force_segments

# The module under test; the mutation test swaps in copies with a planted mistake.
OV = oracle.varlen

NAN_BF16 = np.uint16(0x7FC0)


def f64(u16):
    return gi.bf16_bits_to_f32(u16).astype(np.float64).reshape(np.shape(u16))


def packed_inputs(lq, lk, Hq, Hkv, D, seed, extra_rows=0):
    """Head-major packed q [Hq, Nq, D], k/v [Hkv, Nk, D] and their boundaries."""
    cu_q, cu_k = gi.cu_from_lengths(lq), gi.cu_from_lengths(lk)
    nq, nk = int(cu_q[-1]) + extra_rows, int(cu_k[-1]) + extra_rows
    q = gi.normal_bf16(seed, gi.TENSOR_Q, (Hq, nq, D))
    k = gi.normal_bf16(seed, gi.TENSOR_K, (Hkv, nk, D))
    v = gi.normal_bf16(seed, gi.TENSOR_V, (Hkv, nk, D))
    return q, k, v, cu_q, cu_k


def packed_segments(cu_q, cu_k, nq, nk):
    """Sequence id and absolute position of every packed query row and key row."""
    seg_q, pos_q = np.full(nq, -1), np.zeros(nq, dtype=np.int64)
    seg_k, pos_k = np.full(nk, -1), np.zeros(nk, dtype=np.int64)
    for s in range(len(cu_q) - 1):
        lq, lk = cu_q[s + 1] - cu_q[s], cu_k[s + 1] - cu_k[s]
        for i in range(lq):
            seg_q[cu_q[s] + i] = s
            pos_q[cu_q[s] + i] = lk - lq + i
        for j in range(lk):
            seg_k[cu_k[s] + j] = s
            pos_k[cu_k[s] + j] = j
    return seg_q, pos_q, seg_k, pos_k


def assert_rows_match(got, ref, atol=1e-12):
    """Same NaN pattern (rows of no sequence) and equal values elsewhere."""
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_allclose(got[ok], ref[ok], rtol=0, atol=atol)


PACKED_CASES = [
    # lengths of the query chunks, lengths of the key ranges, Hq, Hkv, D, window
    ([5, 3, 7], [5, 3, 7], 4, 2, 8, 0),          # self-attention chunks
    ([2, 4, 1], [6, 4, 9], 4, 1, 8, 0),          # chunks after cached prefixes (MQA)
    ([3, 0, 4], [3, 2, 4], 2, 2, 4, 0),          # an empty query chunk (MHA)
    ([6, 5], [9, 5], 6, 2, 8, 3),                # window, G = 3
    ([1, 1, 1, 1], [4, 1, 7, 2], 4, 2, 8, 0),    # one decode query per sequence
]


@pytest.mark.parametrize("case", PACKED_CASES, ids=[str(c) for c in PACKED_CASES])
def test_packed_matches_segment_mask_matrix_form(case):
    lq, lk, Hq, Hkv, D, w = case
    q, k, v, cu_q, cu_k = packed_inputs(lq, lk, Hq, Hkv, D, seed=51, extra_rows=2)
    out = OV.attention_varlen(q, k, v, len(lq), cu_q=cu_q, cu_k=cu_k, window=w)
    seg = packed_segments(cu_q, cu_k, q.shape[1], k.shape[1])
    ref = brute_force_segments(f64(q), f64(k), f64(v), *seg, window=w)
    assert_rows_match(out, ref)


def test_padded_ignores_padding_and_matches_segment_mask():
    S, Hq, Hkv, D, Tq, Tk = 3, 4, 2, 8, 6, 9
    lq, lk = np.array([6, 2, 4]), np.array([9, 3, 4])
    q = gi.normal_bf16(53, gi.TENSOR_Q, (S, Hq, Tq, D))
    k = gi.normal_bf16(53, gi.TENSOR_K, (S, Hkv, Tk, D))
    v = gi.normal_bf16(53, gi.TENSOR_V, (S, Hkv, Tk, D))
    for s in range(S):  # padding holds NaN: the oracle must never read it
        q[s, :, lq[s]:] = NAN_BF16
        k[s, :, lk[s]:] = NAN_BF16
        v[s, :, lk[s]:] = NAN_BF16
    out = OV.attention_varlen(q, k, v, S, len_q=lq, len_k=lk)
    assert out.shape == q.shape
    # flatten batches onto one token axis; padding rows belong to no sequence
    flat = lambda x: np.ascontiguousarray(x.transpose(1, 0, 2, 3).reshape(x.shape[1], -1, D))
    seg_q = np.array([s if t < lq[s] else -1 for s in range(S) for t in range(Tq)])
    pos_q = np.array([lk[s] - lq[s] + t for s in range(S) for t in range(Tq)])
    seg_k = np.array([s if t < lk[s] else -1 for s in range(S) for t in range(Tk)])
    pos_k = np.array([t for s in range(S) for t in range(Tk)])
    qf, kf, vf = (np.nan_to_num(f64(flat(x)), nan=0.0) for x in (q, k, v))
    ref = brute_force_segments(qf, kf, vf, seg_q, pos_q, seg_k, pos_k)
    got = out.transpose(1, 0, 2, 3).reshape(Hq, -1, D)
    assert_rows_match(got, ref)


def test_packed_queries_over_a_padded_cache():
    lq, lk = np.array([3, 1, 5]), np.array([7, 1, 5])
    Hq, Hkv, D, Tk = 4, 2, 8, 8
    cu_q = gi.cu_from_lengths(lq)
    q = gi.normal_bf16(55, gi.TENSOR_Q, (Hq, int(cu_q[-1]), D))
    k = gi.normal_bf16(55, gi.TENSOR_K, (3, Hkv, Tk, D))
    v = gi.normal_bf16(55, gi.TENSOR_V, (3, Hkv, Tk, D))
    out = OV.attention_varlen(q, k, v, 3, cu_q=cu_q, len_k=lk)
    seg_q = np.repeat(np.arange(3), lq)
    pos_q = np.concatenate([np.arange(lk[s] - lq[s], lk[s]) for s in range(3)])
    seg_k = np.array([s if t < lk[s] else -1 for s in range(3) for t in range(Tk)])
    pos_k = np.tile(np.arange(Tk), 3)
    flat = lambda x: np.ascontiguousarray(x.transpose(1, 0, 2, 3).reshape(Hkv, -1, D))
    ref = brute_force_segments(f64(q), f64(flat(k)), f64(flat(v)), seg_q, pos_q, seg_k, pos_k)
    assert_rows_match(out, ref)


def test_equal_lengths_packed_equals_dense_batch():
    """S sequences of equal length packed head-major are the dense [B, H, T, D] call."""
    B, Hq, Hkv, T, D = 3, 4, 2, 7, 8
    q = gi.normal_bf16(57, gi.TENSOR_Q, (B, Hq, T, D))
    k = gi.normal_bf16(57, gi.TENSOR_K, (B, Hkv, T, D))
    v = gi.normal_bf16(57, gi.TENSOR_V, (B, Hkv, T, D))
    pack = lambda x: np.ascontiguousarray(x.transpose(1, 0, 2, 3).reshape(x.shape[1], B * T, D))
    cu = gi.cu_from_lengths([T] * B)
    out, lse = OV.attention_varlen(pack(q), pack(k), pack(v), B, cu_q=cu, cu_k=cu, with_lse=True)
    ref, ref_lse = oracle.attention(q, k, v, with_lse=True)
    np.testing.assert_array_equal(out, pack(ref))
    np.testing.assert_array_equal(lse, ref_lse.transpose(1, 0, 2).reshape(Hq, B * T))


def test_rejects_inconsistent_bounds():
    q, k, v, cu_q, cu_k = packed_inputs([3, 2], [3, 2], 2, 1, 4, seed=59)
    with pytest.raises(ValueError):   # more queries than keys in a sequence
        OV.attention_varlen(q, k, v, 2, cu_q=cu_q, cu_k=np.array([0, 2, 5], dtype=np.int32))
    with pytest.raises(ValueError):   # boundaries not non-decreasing
        OV.attention_varlen(q, k, v, 2, cu_q=np.array([0, 4, 3], dtype=np.int32), cu_k=cu_k)
    with pytest.raises(ValueError):   # past the rows
        OV.attention_varlen(q, k, v, 2, cu_q=cu_q, cu_k=np.array([0, 3, 9], dtype=np.int32))


def test_gather_pages_matches_an_element_loop():
    P, H, page, D = 7, 2, 4, 3
    pool = gi.normal_bf16(61, gi.TENSOR_K, (P, H, page, D))
    table = np.array([[5, 0, 3], [6, 2, -1]], dtype=np.int32)
    lens = np.array([10, 6])
    got = OV.gather_pages(pool, table, lens, page)
    assert got.shape == (2, H, 10, D)
    for b in range(2):
        for h in range(H):
            for t in range(10):
                want = pool[table[b, t // page], h, t % page] if t < lens[b] else np.zeros(D, np.uint16)
                np.testing.assert_array_equal(got[b, h, t], want)


def test_paged_cache_decode_equals_contiguous_cache():
    """A cache cut into pages and stored in a shuffled pool gives the same decode."""
    B, Hq, Hkv, D, page, Tq = 3, 8, 2, 8, 4, 2
    lens = np.array([13, 2, 8])
    T = int(lens.max())
    q = gi.normal_bf16(63, gi.TENSOR_Q, (B, Hq, Tq, D))
    k = gi.normal_bf16(63, gi.TENSOR_K, (B, Hkv, T, D))
    v = gi.normal_bf16(63, gi.TENSOR_V, (B, Hkv, T, D))
    n_pages = (lens + page - 1) // page
    order = gi.permutation(63, gi.STREAM_PAGES, int(n_pages.sum()))
    table = np.full((B, int(n_pages.max())), -1, dtype=np.int32)
    kp = np.zeros((order.size, Hkv, page, D), np.uint16)
    vp = np.zeros_like(kp)
    at = 0
    for b in range(B):
        for i in range(n_pages[b]):
            pg = order[at]
            at += 1
            table[b, i] = pg
            rows = slice(i * page, min((i + 1) * page, lens[b]))
            n = rows.stop - rows.start
            kp[pg, :, :n] = k[b, :, rows]
            vp[pg, :, :n] = v[b, :, rows]
    kc = OV.gather_pages(kp, table, lens, page)
    vc = OV.gather_pages(vp, table, lens, page)
    got = OV.attention_varlen(q, kc, vc, B, len_k=lens)
    for b in range(B):
        ref = oracle.attention(q[b:b + 1], np.ascontiguousarray(k[b:b + 1, :, :lens[b]]),
                               np.ascontiguousarray(v[b:b + 1, :, :lens[b]]))
        np.testing.assert_array_equal(got[b], ref[0])
