"""GPU parity of the sliding-window forward (gqa_attn_fwd_ex) and of small-T_q decode
chunks with and without a window (gqa_attn_decode_ex), against the fp64 oracle."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import assert_parity, from_dev, rand_qkv, to_dev, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    torch_mod()
    import grouped_query_softmax_b200 as m
    return m


def _sync_ok(gqa):
    torch_mod().cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK


WIN_FWD = [
    # B, Hq, Hkv, Tq, Tk, D, window
    (1, 4, 2, 1000, 1000, 128, 1),       # only the own position
    (1, 4, 2, 1000, 1000, 128, 100),     # window inside one tile, not tile-aligned
    (2, 4, 2, 600, 600, 64, 128),        # tile-aligned window
    (1, 8, 1, 777, 1300, 128, 300),      # MQA, suffix offset 523
    (2, 6, 2, 500, 500, 128, 257),       # odd group size: row-paired sub-tiles
    (1, 2, 2, 300, 1111, 128, 1111),     # window covering everything = causal
    (1, 4, 4, 513, 2048, 128, 1024),     # MHA suffix, long window
]


@pytest.mark.parametrize("case", WIN_FWD, ids=[str(c) for c in WIN_FWD])
def test_window_fwd_matches_oracle(gqa, case):
    B, Hq, Hkv, Tq, Tk, D, w = case
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=41)
    o = gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), window=w)
    _sync_ok(gqa)
    assert_parity(from_dev(o), oracle.attention(q, k, v, window=w), f"window fwd {case}")


def test_window_fwd_lse(gqa):
    q, k, v = rand_qkv(1, 4, 2, 400, 400, 128, seed=42)
    o, lse = gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), window=70, return_lse=True)
    ref, ref_lse = oracle.attention(q, k, v, window=70, with_lse=True)
    assert_parity(from_dev(o), ref, "window fwd lse")
    assert np.abs(lse.cpu().numpy() - ref_lse).max() < 1e-3


CHUNKS = [
    # B, Hq, Hkv, Tq, Tk, D, window, splits
    (2, 8, 2, 2, 1000, 128, 0, 0),
    (4, 32, 8, 4, 4096, 128, 0, 0),      # G*Tq = 16: one full MMA tile per KV head
    (2, 8, 2, 7, 1030, 128, 0, 3),       # last block starts after some rows' positions
    (2, 32, 1, 16, 2000, 64, 0, 0),      # MQA: 512 rows per KV head
    (2, 12, 4, 3, 900, 128, 0, 4),       # G = 3
    (2, 8, 2, 1, 5000, 128, 700, 0),     # plain decode in a window
    (2, 8, 2, 5, 5000, 128, 300, 6),     # chunk in a window, several splits
    (1, 4, 4, 16, 300, 128, 20, 2),      # window shorter than the chunk
]


@pytest.mark.parametrize("case", CHUNKS, ids=[str(c) for c in CHUNKS])
def test_decode_chunk_matches_oracle(gqa, case):
    B, Hq, Hkv, Tq, Tk, D, w, splits = case
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=43)
    o = gqa.attn_decode(to_dev(q), to_dev(k), to_dev(v), window=w, num_splits=splits)
    _sync_ok(gqa)
    assert_parity(from_dev(o), oracle.attention(q, k, v, window=w), f"decode chunk {case}")


def test_decode_chunk_equals_last_rows_of_prefill(gqa):
    """The pages' suffix check across the two kernels. Each output is rounded to bf16
    once after fp32 sums taken in different orders, so they may differ by about a bf16
    ulp of O(0.1..1) values: max-abs 1e-2, mean-abs 1e-3."""
    q, k, v = rand_qkv(2, 8, 2, 900, 900, 128, seed=44)
    for w in (0, 200):
        full = from_dev(gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), window=w))
        for tq in (1, 4, 16):
            part = gqa.attn_decode(to_dev(np.ascontiguousarray(q[:, :, -tq:])), to_dev(k), to_dev(v), window=w)
            _sync_ok(gqa)
            assert_parity(from_dev(part), full[:, :, -tq:].astype(np.float64), f"chunk {tq} w {w}",
                          max_abs=1e-2, mean_abs=1e-3)


def test_decode_chunk_rejects_long_chunks_and_negative_windows(gqa):
    P = 1 << 20
    st = gqa.gqa_attn_decode_ex(P, P, P, P, 1, 4, 2, 17, 100, 64, 2 * 100 * 64, 100 * 64, 2 * 100 * 64,
                                100 * 64, 0.0, 0, 1, None, 0, None)
    assert st == gqa.GQA_ERR_UNSUPPORTED
    st = gqa.gqa_attn_decode_ex(P, P, P, P, 1, 4, 2, 2, 100, 64, 2 * 100 * 64, 100 * 64, 2 * 100 * 64,
                                100 * 64, 0.0, -1, 1, None, 0, None)
    assert st == gqa.GQA_ERR_INVALID_ARGUMENT
