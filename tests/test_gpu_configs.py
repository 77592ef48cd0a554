"""Parity at the benchmark workloads' full sizes, in the launch configuration bench.py
times (gqa_attn_fwd for prefill and suffix, gqa_attn_decode with automatic splits).

The GPU computes every output; the fp64 oracle checks all rows where that takes
seconds (tiny, GQA decode, MHA suffix) and a seeded sample of at least 4096 rows
plus the special rows (i = 0, tile boundaries +-1, the last row, every (b, a)) for
the two long prefill workloads. Rows are independent, so every sampled row is
checked exactly against its own fp64 value.
"""
import numpy as np
import pytest

import gqa_inputs as gi
import oracle
from tests.gpu_util import assert_parity, bits_of, sample_rows, to_dev, torch_mod

pytestmark = pytest.mark.gpu


def _rows_to_f32(bits_flat, rows, D):
    return gi.bf16_bits_to_f32(bits_flat.reshape(-1, D)[rows]).astype(np.float64)


@pytest.mark.parametrize("name", ["tiny", "gqa_prefill", "mqa_long", "mha_suffix", "swa_prefill"])
def test_prefill_workload_full_size(name):
    torch = torch_mod()
    import grouped_query_softmax_b200 as gqa
    w = gi.WORKLOADS[name]
    q, k, v = w.make()
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o = gqa.attn_fwd(qd, kd, vd, window=w.window)
    torch.cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    out_bits = bits_of(o)
    total = w.B * w.Hq * w.Tq
    if total <= 65536:
        rows = np.arange(total)
    else:
        rows = sample_rows(w.B, w.Hq, w.Tq, 4096, seed=1)
        assert len(rows) >= 4096
    ref = oracle.attention_rows(q, k, v, rows, window=w.window)
    assert_parity(_rows_to_f32(out_bits, rows, w.D), ref, f"{name} ({len(rows)} rows)")
    if name == "gqa_prefill":
        # run-to-run determinism of the full output
        o2 = gqa.attn_fwd(qd, kd, vd)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bits_of(o2), out_bits)


@pytest.mark.parametrize("name", ["gqa_decode", "chunk_decode"])
def test_decode_workload_full_size(name):
    torch = torch_mod()
    import grouped_query_softmax_b200 as gqa
    w = gi.WORKLOADS[name]                   # B64 Hq32 Hkv8, 32768 cached keys: 8 GiB of K/V
    q, k, v = w.make()
    kd = to_dev(k)
    vd = to_dev(v)
    qd = to_dev(q)
    o = gqa.attn_decode(qd, kd, vd, window=w.window)   # automatic split count, as the bench runs it
    torch.cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    rows = np.arange(w.B * w.Hq * w.Tq)
    ref = oracle.attention_rows(q, k, v, rows, window=w.window)
    assert_parity(_rows_to_f32(bits_of(o), rows, w.D), ref, f"{name} (all rows)")
