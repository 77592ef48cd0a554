"""gqa_attn_decode_static: decode without a caller workspace.

Some callers cannot allocate device memory when they call decode: a plugin inside
an inference engine that owns every byte of device memory, or a latency-critical
decode loop where cudaMalloc (which can synchronise the device) is not allowed.
For them the library offers gqa_attn_decode_static, which keeps its split-KV
partials in a fixed 16 MiB scratch array compiled into the library instead of a
workspace the caller would have to allocate. These tests call it through the C ABI
and check it against the ordinary workspace entry point.

This file is named to be collected last: it must pass on its own in a fresh process
and after every other test.
"""
import numpy as np
import pytest

from tests.gpu_util import MAX_ABS, MEAN_ABS, assert_parity, bits_of, from_dev, rand_qkv, to_dev, torch_mod

pytestmark = pytest.mark.gpu


def _decode_static(gqa, qd, kd, vd, od, B, Hq, Hkv, Tk, D, num_splits):
    torch = torch_mod()
    return gqa.gqa_attn_decode_static(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                                      B, Hq, Hkv, Tk, D, kd.stride(0), kd.stride(1), vd.stride(0),
                                      vd.stride(1), 0.0, num_splits,
                                      torch.cuda.current_stream().cuda_stream)


def test_static_scratch_decode_matches_workspace_decode_on_two_calls():
    """The same kernels with the same split count on the same inputs: the static call's
    output equals the workspace call's bit for bit, on two calls in a row, and the
    second call leaves the device's free memory unchanged (it allocates nothing)."""
    torch = torch_mod()
    import grouped_query_softmax_b200 as gqa
    B, Hq, Hkv, Tk, D = 8, 32, 8, 4096, 128
    assert gqa.gqa_attn_decode_num_splits(B, Hq, Hkv, Tk, D, 0) > 1   # the scratch is really used
    for call, seed in enumerate((31, 32)):                            # two calls in a row
        q, k, v = rand_qkv(B, Hq, Hkv, 1, Tk, D, seed=seed)
        qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
        ref = gqa.attn_decode(qd, kd, vd)                              # workspace entry point
        od = torch.full_like(qd, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        st = _decode_static(gqa, qd, kd, vd, od, B, Hq, Hkv, Tk, D, 0)
        assert st == gqa.GQA_OK, gqa.gqa_status_string(st)
        torch.cuda.synchronize()
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free_before
        assert gqa.gqa_get_device_error() == gqa.GQA_OK
        assert np.array_equal(bits_of(od), bits_of(ref)), f"static decode call {call} differs from the workspace call"
        assert_parity(from_dev(od), from_dev(ref).astype(np.float64), f"static decode call {call}",
                      max_abs=MAX_ABS, mean_abs=MEAN_ABS)


def test_static_decode_with_one_split_writes_o_directly():
    """num_splits = 1 uses no scratch; the result still equals the workspace call's."""
    torch = torch_mod()
    import grouped_query_softmax_b200 as gqa
    B, Hq, Hkv, Tk, D = 2, 8, 2, 1000, 64
    q, k, v = rand_qkv(B, Hq, Hkv, 1, Tk, D, seed=33)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    ref = gqa.attn_decode(qd, kd, vd, num_splits=1)
    od = torch.full_like(qd, float("nan"))
    st = _decode_static(gqa, qd, kd, vd, od, B, Hq, Hkv, Tk, D, 1)
    assert st == gqa.GQA_OK, gqa.gqa_status_string(st)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(od), bits_of(ref))


def test_static_scratch_rejects_problems_larger_than_the_scratch():
    import grouped_query_softmax_b200 as gqa
    B, Hq, Hkv, Tk, D, splits = 64, 64, 8, 8192, 128, 8        # 8*64*64*(128+1)*4 B > 16 MiB
    assert gqa.gqa_attn_decode_workspace_bytes(B, Hq, Hkv, Tk, D, splits) > 16 << 20
    fake = 1 << 20                                              # never dereferenced: rejected first
    st = gqa.gqa_attn_decode_static(fake, fake, fake, fake, B, Hq, Hkv, Tk, D, Hkv * Tk * D, Tk * D,
                                    Hkv * Tk * D, Tk * D, 0.0, splits, None)
    assert st == gqa.GQA_ERR_WORKSPACE
