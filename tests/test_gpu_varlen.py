"""GPU parity of sequences of different lengths: packed / padded forward
(gqa_attn_fwd_varlen) and decode over per-sequence cache lengths, contiguous or paged
(gqa_attn_decode_varlen), against the fp64 oracle's packed, padded and paged forms.

Padding, unused page rows and unused pool pages are filled with NaN bit patterns: a
kernel that lets any of them into a valid row (0 * NaN in P V) fails the finite check.
"""
import numpy as np
import pytest

import gqa_inputs as gi
import oracle
import oracle.varlen as ov
from tests.gpu_util import assert_parity, bits_of, from_dev, to_dev, torch_mod

pytestmark = pytest.mark.gpu

NAN_BITS = np.uint16(0x7FC0)


@pytest.fixture(scope="module")
def gqa():
    torch_mod()
    import grouped_query_softmax_b200 as m
    return m


def _sync_ok(gqa):
    torch_mod().cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK


def _i32(x):
    torch = torch_mod()
    return torch.tensor(np.asarray(x, dtype=np.int32), device="cuda")


def _packed(lq, lk, Hq, Hkv, D, seed, extra=0):
    """Token-major packed q [Nq, Hq, D], k/v [Nk, Hkv, D] (+ `extra` NaN rows at the end)."""
    cu_q, cu_k = gi.cu_from_lengths(lq), gi.cu_from_lengths(lk)
    nq, nk = int(cu_q[-1]) + extra, int(cu_k[-1]) + extra
    q = gi.normal_bf16(seed, gi.TENSOR_Q, (nq, Hq, D))
    k = gi.normal_bf16(seed, gi.TENSOR_K, (nk, Hkv, D))
    v = gi.normal_bf16(seed, gi.TENSOR_V, (nk, Hkv, D))
    if extra:
        q[-extra:] = NAN_BITS
        k[-extra:] = NAN_BITS
        v[-extra:] = NAN_BITS
    return q, k, v, cu_q, cu_k


def _head_major(x):
    return np.ascontiguousarray(x.transpose(1, 0, 2))


def _check_packed(got_tok, ref_head_major, cu_q, what):
    """got: token-major [Nq, Hq, D] float; ref: head-major [Hq, Nq, D] with NaN off-sequence."""
    rows = np.arange(int(cu_q[-1]))
    got = got_tok.transpose(1, 0, 2)[:, rows]
    ref = ref_head_major[:, rows]
    assert not np.isnan(ref).any()
    assert_parity(got, ref, what)


PACKED = [
    # query chunk lengths, key lengths, Hq, Hkv, D, window
    ([1000, 37, 128, 129, 255, 700], None, 8, 2, 128, 0),         # self-attention, ragged tails
    ([300, 0, 513, 64], [1800, 5, 513, 1000], 8, 2, 128, 0),      # chunks after cached prefixes, one empty
    ([640, 200, 900], None, 6, 2, 128, 0),                        # odd group size: row-paired units
    ([777, 1300], [900, 1300], 8, 1, 128, 300),                   # MQA with a window
    ([520, 61, 384], [600, 61, 1000], 4, 4, 64, 0),               # MHA, D = 64
]


@pytest.mark.parametrize("case", PACKED, ids=[str(c[:2]) for c in PACKED])
def test_packed_token_major_matches_oracle(gqa, case):
    lq, lk, Hq, Hkv, D, w = case
    lk = lq if lk is None else lk
    q, k, v, cu_q, cu_k = _packed(lq, lk, Hq, Hkv, D, seed=71, extra=100)
    o, lse = gqa.attn_fwd_varlen(to_dev(q), to_dev(k), to_dev(v), cu_seqlens_q=_i32(cu_q),
                                 cu_seqlens_k=_i32(cu_k), window=w, return_lse=True)
    _sync_ok(gqa)
    ref, ref_lse = ov.attention_varlen(_head_major(q), _head_major(k), _head_major(v), len(lq),
                                       cu_q=cu_q, cu_k=cu_k, window=w, with_lse=True)
    _check_packed(from_dev(o), ref, cu_q, f"packed {case[:2]}")
    n = int(cu_q[-1])
    assert np.abs(lse.cpu().numpy()[:, :n] - ref_lse[:, :n]).max() < 1e-3


def test_packed_head_major_and_untouched_rows(gqa):
    torch = torch_mod()
    lq = [300, 129, 1]
    q, k, v, cu_q, cu_k = _packed(lq, lq, 8, 2, 128, seed=73, extra=7)
    qh, kh, vh = (to_dev(_head_major(x)) for x in (q, k, v))
    # [H, rows, D] buffers passed as [rows, H, D] views (head stride rows*D, row stride D)
    out = torch.full_like(qh, 3.0)
    o = gqa.attn_fwd_varlen(qh.transpose(0, 1), kh.transpose(0, 1), vh.transpose(0, 1),
                            cu_seqlens_q=_i32(cu_q), cu_seqlens_k=_i32(cu_k), out=out.transpose(0, 1))
    _sync_ok(gqa)
    ref = ov.attention_varlen(_head_major(q), _head_major(k), _head_major(v), 3, cu_q=cu_q, cu_k=cu_k)
    got = from_dev(out)
    n = int(cu_q[-1])
    assert_parity(got[:, :n], ref[:, :n], "head-major packed")
    assert (got[:, n:] == 3.0).all(), "rows of no sequence were written"


def test_padded_with_nan_padding_matches_oracle(gqa):
    S, Hq, Hkv, D, Tq, Tk = 4, 8, 2, 128, 700, 1100
    lq, lk = np.array([700, 1, 333, 129]), np.array([1100, 1, 333, 900])
    q = gi.normal_bf16(75, gi.TENSOR_Q, (S, Hq, Tq, D))
    k = gi.normal_bf16(75, gi.TENSOR_K, (S, Hkv, Tk, D))
    v = gi.normal_bf16(75, gi.TENSOR_V, (S, Hkv, Tk, D))
    for s in range(S):
        q[s, :, lq[s]:] = NAN_BITS
        k[s, :, lk[s]:] = NAN_BITS
        v[s, :, lk[s]:] = NAN_BITS
    o = gqa.attn_fwd_varlen(to_dev(q), to_dev(k), to_dev(v), seqlens_q=_i32(lq), seqlens_k=_i32(lk))
    _sync_ok(gqa)
    ref = ov.attention_varlen(q, k, v, S, len_q=lq, len_k=lk)
    got = from_dev(o)
    for s in range(S):
        assert_parity(got[s, :, :lq[s]], ref[s, :, :lq[s]], f"padded sequence {s}")


def test_packed_chunks_over_a_padded_cache(gqa):
    """Chunked prefill: new tokens packed, keys read from a per-sequence padded cache."""
    lq, lk = np.array([200, 64, 513]), np.array([1000, 64, 2000])
    Hq, Hkv, D, T = 8, 2, 128, 2048
    cu_q = gi.cu_from_lengths(lq)
    q = gi.normal_bf16(77, gi.TENSOR_Q, (int(cu_q[-1]), Hq, D))
    k = gi.normal_bf16(77, gi.TENSOR_K, (3, Hkv, T, D))
    v = gi.normal_bf16(77, gi.TENSOR_V, (3, Hkv, T, D))
    for s in range(3):
        k[s, :, lk[s]:] = NAN_BITS
        v[s, :, lk[s]:] = NAN_BITS
    o = gqa.attn_fwd_varlen(to_dev(q), to_dev(k), to_dev(v), cu_seqlens_q=_i32(cu_q), seqlens_k=_i32(lk))
    _sync_ok(gqa)
    ref = ov.attention_varlen(_head_major(q), k, v, 3, cu_q=cu_q, len_k=lk)
    _check_packed(from_dev(o), ref, cu_q, "packed over padded")


def test_equal_lengths_match_the_dense_kernel_bitwise(gqa):
    """Same tiles, same order inside every row: the two launches agree bit for bit."""
    B, Hq, Hkv, T, D = 3, 8, 2, 600, 128
    q = gi.normal_bf16(79, gi.TENSOR_Q, (B, Hq, T, D))
    k = gi.normal_bf16(79, gi.TENSOR_K, (B, Hkv, T, D))
    v = gi.normal_bf16(79, gi.TENSOR_V, (B, Hkv, T, D))
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    dense = gqa.attn_fwd(qd, kd, vd)
    padded = gqa.attn_fwd_varlen(qd, kd, vd)                    # padded form, every row valid
    cu = _i32(gi.cu_from_lengths([T] * B))
    tok = lambda t: t.transpose(1, 2).reshape(B * T, t.shape[1], D)  # token-major copies
    packed = gqa.attn_fwd_varlen(tok(qd), tok(kd), tok(vd), cu_seqlens_q=cu, cu_seqlens_k=cu)
    _sync_ok(gqa)
    np.testing.assert_array_equal(bits_of(padded), bits_of(dense))
    np.testing.assert_array_equal(bits_of(packed), bits_of(tok(dense)))


def test_bad_sequence_bounds_are_reported_and_nothing_is_written(gqa):
    torch = torch_mod()
    q, k, v, cu_q, cu_k = _packed([100, 50], [100, 50], 4, 2, 64, seed=81)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    bad_cases = [
        (np.array([0, 100, 160], np.int32), cu_k),   # past the query rows
        (cu_q, np.array([0, 100, 120], np.int32)),   # more queries than keys (50 > 20)
        (np.array([0, 120, 150], np.int32), np.array([0, 100, 150], np.int32)),  # 120 > 100 keys
    ]
    for bq, bk in bad_cases:
        out = torch.full_like(qd, 5.0)
        gqa.attn_fwd_varlen(qd, kd, vd, cu_seqlens_q=_i32(bq), cu_seqlens_k=_i32(bk), max_seqlen_q=150,
                            out=out)
        torch.cuda.synchronize()
        assert gqa.gqa_get_device_error() == gqa.GQA_ERR_INVALID_ARGUMENT
        assert (from_dev(out) == 5.0).all()
    # the context is still good: a correct call works afterwards
    o = gqa.attn_fwd_varlen(qd, kd, vd, cu_seqlens_q=_i32(cu_q), cu_seqlens_k=_i32(cu_k))
    _sync_ok(gqa)
    ref = ov.attention_varlen(_head_major(q), _head_major(k), _head_major(v), 2, cu_q=cu_q, cu_k=cu_k)
    _check_packed(from_dev(o), ref, cu_q, "after bad bounds")


def test_full_size_varlen_workloads(gqa):
    """The bench's packed workloads at full size, checked on a seeded row sample."""
    for name in ("varlen_prefill", "chunked_prefill"):
        w = gi.VARLEN_WORKLOADS[name]
        q, k, v, cu_q, cu_k = w.make()
        o = gqa.attn_fwd_varlen(to_dev(q), to_dev(k), to_dev(v), cu_seqlens_q=_i32(cu_q),
                                cu_seqlens_k=_i32(cu_k))
        _sync_ok(gqa)
        got = from_dev(o)
        rng = np.random.default_rng(5)
        seqs = sorted(set(rng.integers(0, w.S, 6).tolist()) | {0, w.S - 1})
        for s in seqs:
            lq_s = int(cu_q[s + 1] - cu_q[s])
            rows = np.unique(np.concatenate([rng.integers(0, lq_s, 24), [0, lq_s - 1]]))
            qs = np.ascontiguousarray(q[cu_q[s]:cu_q[s + 1]].transpose(1, 0, 2)[None])
            ks = np.ascontiguousarray(k[cu_k[s]:cu_k[s + 1]].transpose(1, 0, 2)[None])
            vs = np.ascontiguousarray(v[cu_k[s]:cu_k[s + 1]].transpose(1, 0, 2)[None])
            flat = np.array([a * lq_s + r for a in range(w.Hq) for r in rows])
            ref = oracle.attention_rows(qs, ks, vs, flat).reshape(w.Hq, len(rows), w.D)
            mine = got[cu_q[s] + rows].transpose(1, 0, 2)
            assert_parity(mine, ref, f"{name} sequence {s}")


# ---------------------------------------------------------------- decode
def _paged_pool(k_cont, v_cont, lens, page, seed, layout="NHD"):
    """Cut a contiguous [B, H, T, D] cache into a shuffled pool; NaN in unused rows/pages."""
    B, H, _, D = k_cont.shape
    n_pages = (lens + page - 1) // page
    spare = 3
    order = gi.permutation(seed, gi.STREAM_PAGES, int(n_pages.sum()) + spare)
    pool_k = np.full((order.size, H, page, D), NAN_BITS, np.uint16)
    pool_v = np.full_like(pool_k, NAN_BITS)
    table = np.full((B, int(n_pages.max()) + 2), -1, np.int32)
    at = 0
    for b in range(B):
        for i in range(n_pages[b]):
            pg = order[at]
            at += 1
            table[b, i] = pg
            r0, r1 = i * page, min((i + 1) * page, lens[b])
            pool_k[pg, :, :r1 - r0] = k_cont[b, :, r0:r1]
            pool_v[pg, :, :r1 - r0] = v_cont[b, :, r0:r1]
    if layout == "NHD":
        pool_k = np.ascontiguousarray(pool_k.transpose(0, 2, 1, 3))
        pool_v = np.ascontiguousarray(pool_v.transpose(0, 2, 1, 3))
    return pool_k, pool_v, table


DECODE = [
    # B, Hq, Hkv, Tq, lengths, D, window, splits, page (0 = contiguous), pool layout
    (4, 8, 2, 1, [5000, 1, 129, 3000], 128, 0, 0, 0, None),
    (3, 8, 2, 4, [700, 4, 2048], 128, 0, 3, 0, None),
    (3, 32, 8, 1, [4100, 300, 2049], 128, 0, 0, 16, "NHD"),
    (3, 8, 2, 2, [1000, 64, 3333], 128, 500, 0, 32, "NHD"),
    (2, 8, 1, 1, [5000, 4097], 128, 0, 5, 64, "HND"),
    (3, 12, 4, 3, [900, 3, 2500], 64, 0, 0, 128, "NHD"),
    (2, 8, 2, 1, [1000, 2600], 128, 0, 0, 256, "NHD"),
]


@pytest.mark.parametrize("case", DECODE, ids=[str(c) for c in DECODE])
def test_decode_varlen_matches_oracle(gqa, case):
    B, Hq, Hkv, Tq, lens, D, w, splits, page, layout = case
    lens = np.array(lens)
    T = int(lens.max())
    q = gi.normal_bf16(83, gi.TENSOR_Q, (B, Hq, Tq, D))
    k = gi.normal_bf16(83, gi.TENSOR_K, (B, Hkv, T, D))
    v = gi.normal_bf16(83, gi.TENSOR_V, (B, Hkv, T, D))
    for b in range(B):
        k[b, :, lens[b]:] = NAN_BITS
        v[b, :, lens[b]:] = NAN_BITS
    if page == 0:
        o = gqa.attn_decode_varlen(to_dev(q), to_dev(k), to_dev(v), _i32(lens), window=w, num_splits=splits)
    else:
        pk, pv, table = _paged_pool(k, v, lens, page, seed=85, layout=layout)
        o = gqa.attn_decode_varlen(to_dev(q), to_dev(pk), to_dev(pv), _i32(lens), block_table=_i32(table),
                                   pool_layout=layout, window=w, num_splits=splits)
    _sync_ok(gqa)
    ref = ov.attention_varlen(q, k, v, B, len_k=lens, window=w)
    assert_parity(from_dev(o), ref, f"decode {case}")


def test_decode_varlen_bad_lengths_are_reported(gqa):
    torch = torch_mod()
    q = gi.normal_bf16(87, gi.TENSOR_Q, (2, 4, 2, 64))
    k = gi.normal_bf16(87, gi.TENSOR_K, (2, 2, 300, 64))
    for lens in ([300, 1], [301, 5], [-3, 10]):   # Tq = 2 > 1; past capacity 300; negative
        gqa.attn_decode_varlen(to_dev(q), to_dev(k), to_dev(k), _i32(lens), num_splits=1)
        torch.cuda.synchronize()
        assert gqa.gqa_get_device_error() == gqa.GQA_ERR_INVALID_ARGUMENT
    o = gqa.attn_decode_varlen(to_dev(q), to_dev(k), to_dev(k), _i32([300, 2]))
    _sync_ok(gqa)
    ref = ov.attention_varlen(q, k, k, 2, len_k=np.array([300, 2]))
    assert_parity(from_dev(o), ref, "decode after bad lengths")


def test_full_size_paged_decode_workload(gqa):
    w = gi.VARLEN_WORKLOADS["paged_decode"]
    q, kp, vp, lens, table = w.make()
    o = gqa.attn_decode_varlen(to_dev(q), to_dev(kp), to_dev(vp), _i32(lens), block_table=_i32(table))
    _sync_ok(gqa)
    got = from_dev(o)
    # gather a few sequences back out of the pool and check them against the oracle
    rng = np.random.default_rng(7)
    for b in sorted(set(rng.integers(0, w.B, 5).tolist()) | {0}):
        hnd_k = np.ascontiguousarray(kp.transpose(0, 2, 1, 3))
        hnd_v = np.ascontiguousarray(vp.transpose(0, 2, 1, 3))
        kc = ov.gather_pages(hnd_k, table[b:b + 1], lens[b:b + 1], w.page)
        vc = ov.gather_pages(hnd_v, table[b:b + 1], lens[b:b + 1], w.page)
        ref = oracle.attention(np.ascontiguousarray(q[b:b + 1]), kc, vc)
        assert_parity(got[b:b + 1], ref, f"paged decode sequence {b}")


PAGED_PREFILL = [
    # chunk lengths, cached-prefix lengths, Hq, Hkv, D, page, pool layout, window
    ([300, 1, 640], [700, 0, 1000], 8, 2, 128, 16, "NHD", 0),
    ([129, 512], [127, 1500], 8, 1, 128, 64, "HND", 0),
    ([700, 200, 33], [0, 900, 4000], 6, 2, 128, 256, "NHD", 300),
    ([257, 100], [600, 77], 4, 4, 64, 128, "NHD", 0),
]


@pytest.mark.parametrize("case", PAGED_PREFILL, ids=[str(c) for c in PAGED_PREFILL])
def test_chunked_prefill_over_a_paged_cache(gqa, case):
    """New tokens packed, every sequence's keys (its cached prefix and the chunk itself)
    in a shuffled page pool; rest-of-page rows and spare pages hold NaN."""
    lq, pre, Hq, Hkv, D, page, layout, w = case
    lq, lk = np.array(lq), np.array(pre) + np.array(lq)
    S, T = len(lq), int(lk.max())
    cu_q = gi.cu_from_lengths(lq)
    q = gi.normal_bf16(89, gi.TENSOR_Q, (int(cu_q[-1]), Hq, D))
    k = gi.normal_bf16(89, gi.TENSOR_K, (S, Hkv, T, D))
    v = gi.normal_bf16(89, gi.TENSOR_V, (S, Hkv, T, D))
    for s in range(S):
        k[s, :, lk[s]:] = NAN_BITS
        v[s, :, lk[s]:] = NAN_BITS
    pk, pv, table = _paged_pool(k, v, lk, page, seed=91, layout=layout)
    o = gqa.attn_fwd_varlen(to_dev(q), to_dev(pk), to_dev(pv), cu_seqlens_q=_i32(cu_q), seqlens_k=_i32(lk),
                            block_table=_i32(table), pool_layout=layout, window=w)
    _sync_ok(gqa)
    ref = ov.attention_varlen(_head_major(q), k, v, S, cu_q=cu_q, len_k=lk, window=w)
    _check_packed(from_dev(o), ref, cu_q, f"paged prefill {case}")


@pytest.mark.parametrize("S, q_hi, k_extra_hi", [
    (40, 700, 1500),    # few sequences: units listed sequence-major and fetched dynamically
    (1100, 4, 6),       # more sequences than the dynamic plan takes: the static longest-first order
])
def test_every_unit_computed_once(gqa, S, q_hi, k_extra_hi):
    """The output starts as NaN: every row of every sequence must be written, by the unit that
    owns it, and a second launch must give the same bits (the CTA that takes a unit varies in a
    dynamically fetched launch, its result must not)."""
    torch = torch_mod()
    lq = gi.uniform_ints(5, gi.STREAM_LEN, S, 1, q_hi)
    lk = lq + gi.uniform_ints(5, gi.STREAM_PREFIX, S, 0, k_extra_hi)
    Hq, Hkv, D = 8, 2, 128
    q, k, v, cu_q, cu_k = _packed(lq, lk, Hq, Hkv, D, seed=77)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    outs = []
    for _ in range(2):
        out = torch.full_like(qd, float("nan"))
        gqa.attn_fwd_varlen(qd, kd, vd, cu_seqlens_q=_i32(cu_q), cu_seqlens_k=_i32(cu_k), out=out)
        _sync_ok(gqa)
        outs.append(bits_of(out))
    assert np.array_equal(outs[0], outs[1])
    got = gi.bf16_bits_to_f32(outs[0]).reshape(q.shape)
    ref = ov.attention_varlen(_head_major(q), _head_major(k), _head_major(v), S, cu_q=cu_q, cu_k=cu_k)
    _check_packed(got, ref, cu_q, f"{S} sequences")
