"""GPU parity of the backward pass (gqa_attn_bwd) against the fp64 oracle's gradients.

The bar is relative to each gradient tensor's own size, because the gradients sum many
terms of both signs: for each of dQ, dK, dV,
    max |gpu - ref|  <= 2^-6 * max |ref|   and   mean |gpu - ref| <= 2^-8 * mean |ref|.
The kernel rounds P, dS and each output to bf16 once (relative error 2^-9 each) and
takes D_i = <dO_i, O_i> from the bf16 forward output; everything else accumulates in fp32.
"""
import numpy as np
import pytest

import gqa_inputs as gi
import oracle
from tests.gpu_util import bits_of, from_dev, to_dev, torch_mod

pytestmark = pytest.mark.gpu

MAX_REL = 2.0 ** -6
MEAN_REL = 2.0 ** -8


@pytest.fixture(scope="module")
def gqa():
    torch_mod()
    import grouped_query_softmax_b200 as m
    return m


def assert_grad_parity(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite gradient"
    err = np.abs(got - ref)
    mx, mean = float(err.max()), float(err.mean())
    scale_max, scale_mean = float(np.abs(ref).max()), float(np.abs(ref).mean())
    assert mx <= MAX_REL * scale_max and mean <= MEAN_REL * scale_mean, (
        f"{what}: max-abs {mx:.3e} (bar {MAX_REL * scale_max:.3e}), mean-abs {mean:.3e} "
        f"(bar {MEAN_REL * scale_mean:.3e})")


def run_bwd(gqa, q, k, v, do):
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse = gqa.attn_fwd(qd, kd, vd, return_lse=True)
    dq, dk, dv = gqa.attn_bwd(qd, kd, vd, o, dod, lse)
    torch_mod().cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    return dq, dk, dv


CASES = [
    # B, Hq, Hkv, Tq, Tk, D
    (1, 4, 2, 128, 128, 64),       # one tile
    (2, 8, 2, 300, 300, 128),      # ragged tiles, G = 4
    (1, 4, 1, 200, 777, 128),      # MQA suffix: 200 queries after 577 cached keys
    (2, 6, 2, 256, 256, 128),      # G = 3
    (1, 4, 4, 129, 257, 64),       # MHA, D = 64, suffix offset 128
    (1, 8, 2, 1000, 1000, 128),    # several tiles per key block and per query head
    (3, 6, 2, 384, 384, 64),       # 6 (batch, KV head) pairs launched as one chunk, longest blocks first
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_bwd_matches_oracle(gqa, case):
    B, Hq, Hkv, Tq, Tk, D = case
    w = gi.Workload("bwd test", B, Hq, Hkv, Tq, Tk, D, seed=111)
    q, k, v = w.make()
    do = w.make_dout()
    dq, dk, dv = run_bwd(gqa, q, k, v, do)
    rq, rk, rv = oracle.attention_bwd(q, k, v, do)
    assert_grad_parity(from_dev(dq), rq, f"dQ {case}")
    assert_grad_parity(from_dev(dk), rk, f"dK {case}")
    assert_grad_parity(from_dev(dv), rv, f"dV {case}")


def test_bwd_key_value_gradients_are_deterministic(gqa):
    w = gi.Workload("bwd det", 1, 8, 2, 512, 512, 128, seed=113)
    q, k, v = w.make()
    do = w.make_dout()
    _, dk1, dv1 = run_bwd(gqa, q, k, v, do)
    _, dk2, dv2 = run_bwd(gqa, q, k, v, do)
    np.testing.assert_array_equal(bits_of(dk1), bits_of(dk2))
    np.testing.assert_array_equal(bits_of(dv1), bits_of(dv2))


def test_bwd_full_size_gqa_prefill(gqa):
    """The GQA prefill workload (B4 Hq32 Hkv8 T4096 D128) on the GPU; batch 0 of every
    gradient checked against the oracle in full (batches are independent)."""
    w = gi.WORKLOADS["gqa_prefill"]
    q, k, v = w.make()
    do = w.make_dout()
    dq, dk, dv = run_bwd(gqa, q, k, v, do)
    b0 = lambda x: np.ascontiguousarray(x[:1])
    rq, rk, rv = oracle.attention_bwd(b0(q), b0(k), b0(v), b0(do))
    assert_grad_parity(from_dev(dq[:1]), rq, "dQ gqa_prefill b0")
    assert_grad_parity(from_dev(dk[:1]), rk, "dK gqa_prefill b0")
    assert_grad_parity(from_dev(dv[:1]), rv, "dV gqa_prefill b0")


WINDOW_CASES = [
    # B, Hq, Hkv, Tq, Tk, D, window
    (1, 4, 2, 700, 700, 128, 200),     # window inside tiles
    (2, 6, 2, 300, 1500, 128, 128),    # suffix far after the prefix: early key blocks unseen (zero grads)
    (1, 8, 1, 513, 513, 64, 8),        # a window much shorter than a tile
]
# Windows of 1 or 2 keys are left to the test below: there dS = P (dP - D) is a difference of
# near-equal terms and D = <dO, O> from the bf16 output carries a rounding error of the same
# size (inherent to forming D from O), so an error bar relative to dQ's own size is too tight.


@pytest.mark.parametrize("case", WINDOW_CASES, ids=[str(c) for c in WINDOW_CASES])
def test_bwd_window_matches_oracle(gqa, case):
    B, Hq, Hkv, Tq, Tk, D, win = case
    w = gi.Workload("bwd window", B, Hq, Hkv, Tq, Tk, D, seed=117)
    q, k, v = w.make()
    do = w.make_dout()
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse = gqa.attn_fwd(qd, kd, vd, window=win, return_lse=True)
    dq, dk, dv = gqa.attn_bwd(qd, kd, vd, o, dod, lse, window=win)
    torch_mod().cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    rq, rk, rv = oracle.attention_bwd(q, k, v, do, window=win)
    assert_grad_parity(from_dev(dq), rq, f"dQ {case}")
    assert_grad_parity(from_dev(dk), rk, f"dK {case}")
    assert_grad_parity(from_dev(dv), rv, f"dV {case}")
    if case[4] - case[3] > 2 * case[6] + 128:
        # keys that no query sees have exactly zero gradients
        unseen = Tk - Tq - win
        assert (from_dev(dk)[:, :, :unseen] == 0).all() and (from_dev(dv)[:, :, :unseen] == 0).all()


def test_bwd_window_of_one_has_no_score_gradient(gqa):
    """With w = 1 every row sees only itself: P = 1, so dS = dP - <dO, o> = 0 exactly and dQ,
    dK vanish; dV_j = dO of the query at position j. A bar relative to a zero reference is
    empty, so dQ and dK are checked against the size of dV instead."""
    w = gi.Workload("bwd window 1", 1, 8, 1, 513, 513, 64, seed=119)
    q, k, v = w.make()
    do = w.make_dout()
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse = gqa.attn_fwd(qd, kd, vd, window=1, return_lse=True)
    dq, dk, dv = gqa.attn_bwd(qd, kd, vd, o, dod, lse, window=1)
    torch_mod().cuda.synchronize()
    assert gqa.gqa_get_device_error() == gqa.GQA_OK
    _, _, rv = oracle.attention_bwd(q, k, v, do, window=1)
    assert_grad_parity(from_dev(dv), rv, "dV window 1")
    scale = float(np.abs(rv).max())
    assert np.abs(from_dev(dq)).max() <= MAX_REL * scale and np.abs(from_dev(dk)).max() <= MAX_REL * scale
