"""GPU parity of gqa_attn_decode (split-KV + log-sum-exp combine) against the oracle."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import assert_parity, bits_of, from_dev, rand_qkv, to_dev, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    torch_mod()
    import grouped_query_softmax_b200 as m
    return m


def run_dec(gqa, q, k, v, **kw):
    torch = torch_mod()
    o = gqa.attn_decode(to_dev(q), to_dev(k), to_dev(v), **kw)
    torch.cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    return o


CASES = [
    # B, Hq, Hkv, Tk, D, splits
    (2, 4, 2, 128, 64, 0),
    (4, 8, 2, 1000, 128, 0),
    (4, 8, 2, 1000, 128, 1),
    (4, 8, 2, 1000, 128, 3),
    (2, 32, 1, 777, 128, 2),      # MQA: 32 heads per KV head -> two 16-head chunks
    (2, 12, 4, 2049, 64, 5),      # G = 3, D = 64
    (1, 2, 2, 1, 128, 0),         # a single cached key
    (3, 40, 2, 300, 128, 0),      # G = 20: a partial 16-head chunk
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_decode_matches_oracle(gqa, case):
    B, Hq, Hkv, Tk, D, splits = case
    q, k, v = rand_qkv(B, Hq, Hkv, 1, Tk, D, seed=11)
    got = from_dev(run_dec(gqa, q, k, v, num_splits=splits))
    assert_parity(got, oracle.attention(q, k, v), f"decode {case}")


def test_decode_equals_last_row_of_prefill(gqa):
    """The pages' suffix check on the GPU: T_q = 1 decode == last row of full causal fwd."""
    q, k, v = rand_qkv(2, 8, 2, 700, 700, 128, seed=12)
    full = from_dev(gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v)))
    last = from_dev(run_dec(gqa, np.ascontiguousarray(q[:, :, -1:]), k, v))
    assert_parity(last, full[:, :, -1:].astype(np.float64), "decode vs fwd", max_abs=1e-2, mean_abs=1e-4)


def test_split_counts_agree(gqa):
    q, k, v = rand_qkv(2, 8, 2, 1, 4096, 128, seed=13)
    ref = oracle.attention(q, k, v)
    outs = [from_dev(run_dec(gqa, q, k, v, num_splits=s)) for s in (1, 2, 7, 32)]
    for o in outs:
        assert_parity(o, ref, "splits")
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 1e-2


def test_decode_deterministic(gqa):
    q, k, v = rand_qkv(4, 8, 2, 1, 3000, 128, seed=14)
    a = bits_of(run_dec(gqa, q, k, v, num_splits=4))
    b = bits_of(run_dec(gqa, q, k, v, num_splits=4))
    np.testing.assert_array_equal(a, b)


def test_decode_strided_cache(gqa):
    torch = torch_mod()
    B, Hq, Hkv, Tk, D, cap = 3, 8, 2, 1500, 128, 2048
    q, k, v = rand_qkv(B, Hq, Hkv, 1, Tk, D, seed=15)
    kc = torch.zeros((B, Hkv, cap, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.full((B, Hkv, cap, D), 9.0, dtype=torch.bfloat16, device="cuda")
    kc[:, :, :Tk] = to_dev(k)
    vc[:, :, :Tk] = to_dev(v)
    o = gqa.attn_decode(to_dev(q), kc, vc, Tk=Tk, num_splits=3)
    assert_parity(from_dev(o), oracle.attention(q, k, v), "strided decode")
