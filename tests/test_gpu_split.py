"""GPU parity of gqa_attn_fwd_split: suffix launches whose last wave of work units is dealt out
over the SMs in runs of key tiles, cut into pieces at unit boundaries and merged by log-sum-exp. Checked against the fp64 oracle, against the unsplit
call, for determinism, and for the workspace rules, all through the C ABI."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import assert_parity, bits_of, from_dev, rand_qkv, to_dev, torch_mod

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, Hq, Hkv, Tq, Tk, D, q_pow2
    (1, 4, 1, 700, 1900, 128, 0),     # MQA-like pair-head units, ragged last row tile
    (2, 16, 16, 512, 4096, 128, 2),   # MHA, peaked softmax (Q x 4)
    (1, 8, 8, 1024, 2048, 128, 0),    # prefix = suffix: some rows see no key in the last part
    (1, 8, 2, 600, 2500, 64, 0),      # D = 64, offset not tile-aligned
    (1, 16, 4, 256, 4096, 128, 0),    # 16 units of 32 key tiles
    (7, 32, 32, 128, 4096, 128, 0),   # a whole wave, then slices crossing unit boundaries;
                                      # one-sub-tile units (T_q = 128)
    (7, 16, 16, 384, 4096, 64, 2),    # the same with D = 64, and units whose second sub-tile is absent
]


@pytest.fixture(scope="module")
def gqa():
    torch_mod()
    import grouped_query_softmax_b200 as m
    return m


def split_call(gqa, qd, kd, vd, Tk, lse=True, workspace="auto"):
    torch = torch_mod()
    B, Hq, Tq, D = qd.shape
    Hkv = kd.shape[1]
    need = gqa.gqa_attn_fwd_split_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, 0)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=qd.device) if workspace == "auto" else workspace
    o = torch.full_like(qd, float("nan"))
    l = torch.full((B, Hq, Tq), float("nan"), dtype=torch.float32, device=qd.device) if lse else None
    st = gqa.gqa_attn_fwd_split(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(),
                                l.data_ptr() if l is not None else None, B, Hq, Hkv, Tq, Tk, D, kd.stride(0),
                                kd.stride(1), vd.stride(0), vd.stride(1), 0.0, 0,
                                ws.data_ptr() if ws is not None else None,
                                ws.numel() if ws is not None else 0, torch.cuda.current_stream().cuda_stream)
    return st, o, l, need


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_split_matches_oracle_and_unsplit(gqa, shape):
    torch = torch_mod()
    B, Hq, Hkv, Tq, Tk, D, qp = shape
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=61, q_pow2=qp)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    st, o, lse, need = split_call(gqa, qd, kd, vd, Tk)
    assert st == gqa.GQA_OK, gqa.gqa_status_string(st)
    torch.cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    assert need > 0, "this shape is expected to split on a B200"
    ref, ref_lse = oracle.attention(q, k, v, with_lse=True)
    assert_parity(from_dev(o), ref, f"split {shape}")
    assert np.abs(lse.cpu().numpy().astype(np.float64) - ref_lse).max() <= 1e-3
    # the unsplit call sums the same keys in another order: the split is no less accurate
    # (mean error against the oracle), and the two differ by no more than their errors allow
    o1, lse1 = gqa.attn_fwd(qd, kd, vd, return_lse=True, split=False)
    got, got1 = from_dev(o).astype(np.float64), from_dev(o1).astype(np.float64)
    err_split, err_unsplit = np.abs(got - ref).mean(), np.abs(got1 - ref).mean()
    assert err_split <= 1.25 * err_unsplit + 1e-6, (err_split, err_unsplit)
    assert np.abs(got - got1).max() <= 2 * max(np.abs(got - ref).max(), np.abs(got1 - ref).max())
    assert np.abs(lse.cpu().numpy() - lse1.cpu().numpy()).max() <= 1e-4
    # fixed merge order: the same bits on a second call
    st, o2, _, _ = split_call(gqa, qd, kd, vd, Tk, lse=False)
    torch.cuda.synchronize()
    assert st == gqa.GQA_OK and np.array_equal(bits_of(o2), bits_of(o))


def test_split_workspace_rules(gqa):
    torch = torch_mod()
    B, Hq, Hkv, Tq, Tk, D = 2, 16, 16, 512, 4096, 128
    q, k, v = rand_qkv(B, Hq, Hkv, Tq, Tk, D, seed=62)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    need = gqa.gqa_attn_fwd_split_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, 0)
    assert need > 0
    big = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    for ws in (None, big[:need - 256], big[16:16 + need]):          # missing, small, misaligned
        st, _, _, _ = split_call(gqa, qd, kd, vd, Tk, lse=False, workspace=ws)
        assert st == gqa.GQA_ERR_WORKSPACE
    # a launch that does not split needs no workspace
    qs, ks, vs = rand_qkv(1, 4, 2, 300, 300, D, seed=63)
    assert gqa.gqa_attn_fwd_split_workspace_bytes(1, 4, 2, 300, 300, D, 0) == 0
    st, o, _, _ = split_call(gqa, to_dev(qs), to_dev(ks), to_dev(vs), 300, lse=False, workspace=None)
    torch.cuda.synchronize()
    assert st == gqa.GQA_OK
    assert_parity(from_dev(o), oracle.attention(qs, ks, vs), "unsplit through gqa_attn_fwd_split")
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
