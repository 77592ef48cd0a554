"""Failure detection on the GPU without faulting it: a bounded wait that nothing
completes runs out, the kernel records GQA_ERR_TIMEOUT and returns, the host reads
the status once, and the context keeps working."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import assert_parity, from_dev, rand_qkv, to_dev, torch_mod

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    torch = torch_mod()
    import grouped_query_softmax_b200 as gqa
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    assert gqa.gqa_selftest_bounded_wait(50_000_000) == gqa.GQA_OK   # 50 ms
    assert gqa.gqa_get_device_error() == gqa.GQA_ERR_TIMEOUT
    assert gqa.gqa_get_device_error() == gqa.GQA_OK                  # read clears it
    q, k, v = rand_qkv(1, 4, 2, 64, 64, 64, seed=20)
    o = gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert_parity(from_dev(o), oracle.attention(q, k, v), "after timeout")
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
