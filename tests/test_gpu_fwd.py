"""GPU parity of gqa_attn_fwd (prefill and suffix) against the fp64 oracle, plus the
invariants the pages and the mathematics fix, all through the C ABI."""
import json
import os

import numpy as np
import pytest

import gqa_inputs as gi
import oracle
from tests.gpu_util import assert_parity, bits_of, from_dev, rand_qkv, to_dev, torch_mod

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def gqa():
    torch_mod()
    import grouped_query_softmax_b200 as m
    return m


def run_fwd(gqa, q, k, v, **kw):
    torch = torch_mod()
    o = gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), **kw)
    torch.cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    return o


SHAPES = [
    # B, Hq, Hkv, Tq, Tk, D
    (2, 4, 2, 128, 128, 64),       # tiny workload
    (1, 2, 1, 129, 129, 64),       # one row past a tile
    (1, 4, 2, 1000, 1000, 128),    # ragged tail, several tiles
    (2, 4, 4, 300, 1111, 128),     # MHA, suffix offset 811 (not tile-aligned)
    (1, 8, 1, 257, 300, 64),       # MQA, offset 43
    (2, 6, 2, 200, 200, 128),      # odd group size 3 -> row-paired sub-tiles
    (1, 1, 1, 1, 1, 64),           # a single key
    (1, 2, 2, 1, 77, 128),         # one query over 77 keys
    (3, 4, 1, 384, 384, 128),      # B=3, three full tiles
    (1, 2, 1, 640, 1280, 64),      # offset 640 (tile-aligned), D=64
]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_fwd_matches_oracle_all_rows(gqa, shape):
    B, Hq, Hkv, Tq, Tk, D = shape
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=1)
    got = from_dev(run_fwd(gqa, q, k, v))
    assert_parity(got, oracle.attention(q, k, v), f"fwd {shape}")


def test_fwd_lse_matches_oracle(gqa):
    q, k, v = rand_qkv(2, 4, 2, 200, 333, 128, seed=2)
    o, lse = gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), return_lse=True)
    ref, ref_lse = oracle.attention(q, k, v, with_lse=True)
    assert_parity(from_dev(o), ref, "fwd with lse")
    err = np.abs(lse.cpu().numpy().astype(np.float64) - ref_lse).max()
    assert err < 1e-3, err


def test_head_mapping_example_embedded_at_d64(gqa):
    """The pages' [1,1,7,7] check, widened to D=64: q = k = 0, v of KV heads 0/1 = 1/7."""
    g = json.load(open(os.path.join(GOLDEN, "head_mapping_example.json")))
    D = 64
    q = np.zeros((1, 4, 1, D), np.uint16)
    k = np.zeros((1, 2, 1, D), np.uint16)
    v = np.stack([gi.f32_to_bf16_bits(np.full((1, D), x, np.float32)) for x in g["v"]]).reshape(1, 2, 1, D)
    got = from_dev(run_fwd(gqa, q, k, v))
    expect = np.repeat(np.array(g["expected_flat"], np.float32), D).reshape(1, 4, 1, D)
    np.testing.assert_array_equal(got, expect)


def test_values_all_ones_give_ones(gqa):
    q, k, _ = rand_qkv(1, 4, 2, 300, 300, 128, seed=3)
    v = gi.f32_to_bf16_bits(np.ones(k.shape, np.float32)).reshape(k.shape)
    got = from_dev(run_fwd(gqa, q, k, v))
    assert_parity(got, np.ones(got.shape), "V = 1")


def test_first_row_sees_only_key_zero(gqa):
    q, k, v = rand_qkv(1, 2, 1, 256, 256, 128, seed=4)
    got = from_dev(run_fwd(gqa, q, k, v))
    np.testing.assert_array_equal(got[:, :, 0], gi.bf16_bits_to_f32(v[:, [0, 0], 0]).reshape(got[:, :, 0].shape))


def test_linear_in_values_bitwise(gqa):
    q, k, v = rand_qkv(1, 4, 2, 256, 256, 64, seed=5)
    v2 = gi.scale_pow2_bf16(v, 1)
    o1 = bits_of(run_fwd(gqa, q, k, v))
    o2 = bits_of(run_fwd(gqa, q, k, v2))
    np.testing.assert_array_equal(o2, gi.scale_pow2_bf16(o1, 1))


def test_gqa_equals_mha_on_repeated_planes_bitwise(gqa):
    for Hkv in (1, 2, 4):
        q, k, v = rand_qkv(1, 8, Hkv, 300, 300, 128, seed=6)
        g = 8 // Hkv
        kr = np.ascontiguousarray(np.repeat(k, g, axis=1))
        vr = np.ascontiguousarray(np.repeat(v, g, axis=1))
        np.testing.assert_array_equal(bits_of(run_fwd(gqa, q, k, v)), bits_of(run_fwd(gqa, q, kr, vr)))


def test_suffix_chunk_equals_rows_of_full_prefill(gqa):
    """fwd(T_q=512 over T_k) equals the last 512 rows of fwd(T_q = T_k)."""
    q, k, v = rand_qkv(1, 4, 2, 1536, 1536, 128, seed=7)
    full = from_dev(run_fwd(gqa, q, k, v))
    for tq in (512, 300, 1):
        part = from_dev(run_fwd(gqa, np.ascontiguousarray(q[:, :, -tq:]), k, v))
        assert_parity(part, full[:, :, -tq:].astype(np.float64), f"suffix {tq}", max_abs=1e-2, mean_abs=1e-4)


def test_strided_cache_slice_equals_contiguous(gqa):
    torch = torch_mod()
    B, Hq, Hkv, Tq, Tk, D, cap = 2, 4, 2, 200, 333, 128, 512
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=8)
    kc = torch.zeros((B, Hkv, cap, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.full((B, Hkv, cap, D), 7.0, dtype=torch.bfloat16, device="cuda")
    kc[:, :, :Tk] = to_dev(k)
    vc[:, :, :Tk] = to_dev(v)
    o_cache = gqa.attn_fwd(to_dev(q), kc, vc, Tk=Tk)
    o_ref = run_fwd(gqa, q, k, v)
    np.testing.assert_array_equal(bits_of(o_cache), bits_of(o_ref))


def test_deterministic_and_no_out_of_bounds_writes(gqa):
    torch = torch_mod()
    B, Hq, Hkv, Tq, Tk, D = 1, 4, 2, 333, 333, 128
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=9)
    n = B * Hq * Tq * D
    guard = 4096
    buf = torch.full((n + 2 * guard,), -3.0, dtype=torch.bfloat16, device="cuda")
    out = buf[guard:guard + n].view(B, Hq, Tq, D)
    gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), out=out)
    first = bits_of(out).copy()
    gqa.attn_fwd(to_dev(q), to_dev(k), to_dev(v), out=out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_of(out), first)
    assert (buf[:guard] == -3.0).all() and (buf[guard + n:] == -3.0).all()


def test_peaked_softmax_stability(gqa):
    """Q scaled by 4 (logits with std ~4), as in the MHA suffix workload."""
    q, k, v = rand_qkv(2, 4, 4, 256, 1024, 128, seed=10, q_pow2=2)
    got = from_dev(run_fwd(gqa, q, k, v))
    assert_parity(got, oracle.attention(q, k, v), "peaked")


def test_boundary_entry_points_by_name(gqa):
    """gqa_attn_fwd and gqa_attn_decode themselves (not their extended siblings), called by
    name through the C ABI with raw device pointers, against the fp64 oracle."""
    torch = torch_mod()
    stream = torch.cuda.current_stream().cuda_stream
    B, Hq, Hkv, Tq, Tk, D = 2, 8, 2, 300, 1111, 128            # suffix offset 811, ragged tiles
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=41)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    od = torch.full_like(qd, float("nan"))
    lse = torch.full((B, Hq, Tq), float("nan"), dtype=torch.float32, device=qd.device)
    st = gqa.gqa_attn_fwd(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(), lse.data_ptr(),
                          B, Hq, Hkv, Tq, Tk, D, kd.stride(0), kd.stride(1), vd.stride(0), vd.stride(1), 0.0, stream)
    assert st == gqa.GQA_OK, gqa.gqa_status_string(st)
    torch.cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    ref, ref_lse = oracle.attention(q, k, v, with_lse=True)
    assert_parity(from_dev(od), ref, "gqa_attn_fwd by name")
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 1e-3

    Bd, Tkd = 4, 5000                                          # decode over several splits
    qd1, kd1, vd1 = rand_qkv(Bd, Hq, Hkv, 1, Tkd, D, seed=42)
    splits = gqa.gqa_attn_decode_num_splits(Bd, Hq, Hkv, Tkd, D, 0)
    assert splits > 1
    need = gqa.gqa_attn_decode_workspace_bytes(Bd, Hq, Hkv, Tkd, D, 0)
    ws = torch.empty(need, dtype=torch.uint8, device=qd.device)
    qq, kk, vv = to_dev(qd1), to_dev(kd1), to_dev(vd1)
    oo = torch.full_like(qq, float("nan"))
    st = gqa.gqa_attn_decode(qq.data_ptr(), kk.data_ptr(), vv.data_ptr(), oo.data_ptr(), Bd, Hq, Hkv, Tkd, D,
                             kk.stride(0), kk.stride(1), vv.stride(0), vv.stride(1), 0.0, 0, ws.data_ptr(), need,
                             stream)
    assert st == gqa.GQA_OK, gqa.gqa_status_string(st)
    torch.cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    assert_parity(from_dev(oo), oracle.attention(qd1, kd1, vd1), "gqa_attn_decode by name")
