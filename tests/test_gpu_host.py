"""GPU tests of gqa_attn_fwd_host (operands in host memory, streamed through a device
workspace in query-row chunks). Each chunk is the suffix call over the keys its rows see, so
the output and the log-sum-exp must equal the one-shot device call bit for bit; one case is
also checked against the fp64 oracle directly."""
import numpy as np
import pytest

import gqa_inputs as gi
import oracle
from tests.gpu_util import assert_parity, to_dev, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    torch_mod()
    import grouped_query_softmax_b200 as m
    return m


def host_bf16(u16, pinned=True):
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pinned else t.clone()


def u16(t):
    torch = torch_mod()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


CASES = [
    # B, Hq, Hkv, Tq, Tk, D, window
    (2, 8, 2, 1000, 1000, 128, 0),    # 4 chunks of 256 rows, the last one ragged
    (1, 4, 1, 700, 1900, 128, 0),     # suffix: 1200 keys before the first query
    (2, 4, 4, 2048, 2048, 64, 0),     # MHA, D = 64, 8 chunks
    (1, 8, 2, 1500, 1500, 128, 300),  # sliding window
    (3, 6, 2, 200, 200, 128, 0),      # a single chunk
    (1, 4, 2, 1, 513, 64, 0),         # one query row
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_host_call_equals_device_call_bitwise(gqa, case):
    B, Hq, Hkv, Tq, Tk, D, win = case
    w = gi.Workload("host test", B, Hq, Hkv, Tq, Tk, D, seed=131)
    q, k, v = w.make()
    o_dev, lse_dev = gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), window=win, return_lse=True, split=False)
    o_host, lse_host = gqa.attn_fwd_host(host_bf16(q), host_bf16(k), host_bf16(v), window=win, return_lse=True)
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    np.testing.assert_array_equal(u16(o_host), u16(o_dev))
    np.testing.assert_array_equal(lse_host.numpy(), lse_dev.cpu().numpy())


def test_host_call_matches_oracle_with_pageable_memory(gqa):
    w = gi.Workload("host oracle", 1, 8, 2, 600, 900, 128, seed=137)
    q, k, v = w.make()
    o = gqa.attn_fwd_host(host_bf16(q, False), host_bf16(k, False), host_bf16(v, False))
    ref = oracle.attention(q, k, v)
    assert_parity(gi.bf16_bits_to_f32(u16(o)).reshape(q.shape), ref, "host call vs oracle")


def test_host_call_full_size_gqa_prefill(gqa):
    w = gi.WORKLOADS["gqa_prefill"]
    q, k, v = w.make()
    o_dev = gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), split=False)
    o_host = gqa.attn_fwd_host(host_bf16(q), host_bf16(k), host_bf16(v))
    np.testing.assert_array_equal(u16(o_host), u16(o_dev))


def test_host_call_error_returns_after_its_queued_copies(gqa):
    """An error after some chunks were queued (forced by the testing hook before chunk 2's
    kernel) returns only once the copies already queued have finished: the output rows of
    chunks 0 and 1 are in host memory when the call returns, with no synchronisation."""
    import ctypes
    lib = ctypes.CDLL(gqa.library_path())
    B, Hq, Hkv, Tq, Tk, D = 2, 8, 2, 2048, 2048, 128          # 8 chunks of 256 rows
    w = gi.Workload("host error path", B, Hq, Hkv, Tq, Tk, D, seed=139)
    q, k, v = w.make()
    o_dev = gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), split=False)
    torch = torch_mod()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    assert lib.gqa_testing_fwd_host_fail_at(2) == 0
    try:
        with pytest.raises(gqa.GqaError):
            gqa.attn_fwd_host(host_bf16(q), host_bf16(k), host_bf16(v), out=out, synchronize=False)
        got = out.view(torch.int16).numpy().view(np.uint16)    # read at once: no synchronisation
        np.testing.assert_array_equal(got[:, :, :512], u16(o_dev)[:, :, :512])
    finally:
        assert lib.gqa_testing_fwd_host_fail_at(-1) == 0
    assert lib.gqa_testing_fwd_host_fail_at(8) == gqa.GQA_ERR_INVALID_ARGUMENT
    o_host = gqa.attn_fwd_host(host_bf16(q), host_bf16(k), host_bf16(v))
    np.testing.assert_array_equal(u16(o_host), u16(o_dev))
