"""Pins for the oracle's backward pass (CPU only).

The gradients are the derivative of the o_a definition, so the main pin is that
derivative taken numerically: central finite differences of the independent matrix-form
forward (tests/brute_force.py) at the same bf16 point, for a seeded set of elements of
Q, K and V, against the oracle's analytic dQ, dK, dV. The other pins are facts of the
mathematics: each row's dS sums to zero, so every column of dK summed over the keys
vanishes; with Q = 0 the weights are uniform, which fixes dV in closed form; GQA's dK and
dV are MHA's on repeated planes summed over the group; and the gradients are linear in dO.
"""
import numpy as np
import pytest

import gqa_inputs as gi
import oracle
from tests.brute_force import brute_force_attention

# the library the pins run against; the mutation test swaps in planted-mistake builds
LIB = None


def bwd(*args, **kw):
    return oracle.attention_bwd(*args, lib=LIB, **kw)


def f64(u16):
    return gi.bf16_bits_to_f32(u16).astype(np.float64).reshape(np.shape(u16))


def inputs(B, Hq, Hkv, Tq, Tk, D, seed):
    w = gi.Workload("bwd pin", B, Hq, Hkv, Tq, Tk, D, seed=seed)
    q, k, v = w.make()
    return q, k, v, w.make_dout()


FD_CASES = [
    # B, Hq, Hkv, Tq, Tk, D, window
    (1, 4, 2, 5, 5, 8, 0),
    (2, 4, 1, 3, 7, 4, 0),      # MQA with a suffix offset
    (1, 6, 3, 6, 6, 8, 3),      # window
]


@pytest.mark.parametrize("case", FD_CASES, ids=[str(c) for c in FD_CASES])
def test_gradients_match_finite_differences_of_the_matrix_form(case):
    B, Hq, Hkv, Tq, Tk, D, w = case
    q, k, v, do = inputs(B, Hq, Hkv, Tq, Tk, D, seed=91)
    qf, kf, vf, dof = f64(q), f64(k), f64(v), f64(do)
    dq, dk, dv = bwd(q, k, v, do, window=w)

    def loss(qx, kx, vx):
        return float(np.sum(dof * brute_force_attention(qx, kx, vx, window=w)))

    rng = np.random.default_rng(3)
    h = 1e-5
    for name, arr, grad in (("q", qf, dq), ("k", kf, dk), ("v", vf, dv)):
        for _ in range(10):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args_p = {"q": (plus, kf, vf), "k": (qf, plus, vf), "v": (qf, kf, plus)}[name]
            args_m = {"q": (minus, kf, vf), "k": (qf, minus, vf), "v": (qf, kf, minus)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-7 + 1e-6 * abs(fd), (name, idx, fd, grad[idx])


def test_key_gradient_columns_sum_to_zero():
    """sum_j dS_ij = 0 for every row, so sum_j dK_j = scale * sum_i (sum_j dS_ij) q_i = 0."""
    for w in (0, 4):
        q, k, v, do = inputs(2, 6, 2, 9, 12, 8, seed=93)
        _, dk, _ = bwd(q, k, v, do, window=w)
        assert np.abs(dk.sum(axis=2)).max() < 1e-12 * max(1.0, np.abs(dk).max())


def test_uniform_weights_give_the_value_gradient_in_closed_form():
    """q = 0: row i weighs its n_i visible keys equally, so dV_j = sum over rows that see j of dO_i / n_i."""
    B, Hq, Hkv, Tq, Tk, D = 1, 4, 2, 4, 6, 8
    q, k, v, do = inputs(B, Hq, Hkv, Tq, Tk, D, seed=95)
    q[...] = 0
    _, dk, dv = bwd(q, k, v, do)
    dof = f64(do)
    want = np.zeros((B, Hkv, Tk, D))
    G = Hq // Hkv
    for a in range(Hq):
        for i in range(Tq):
            pos = Tk - Tq + i
            want[0, a // G, :pos + 1] += dof[0, a, i] / (pos + 1)
    np.testing.assert_allclose(dv, want, rtol=0, atol=1e-13)


def test_gqa_gradients_are_mha_gradients_summed_over_the_group():
    B, Hq, Hkv, Tq, Tk, D = 2, 6, 2, 5, 8, 8
    q, k, v, do = inputs(B, Hq, Hkv, Tq, Tk, D, seed=97)
    G = Hq // Hkv
    dq, dk, dv = bwd(q, k, v, do)
    kr = np.ascontiguousarray(np.repeat(k, G, axis=1))
    vr = np.ascontiguousarray(np.repeat(v, G, axis=1))
    dq_m, dk_m, dv_m = bwd(q, kr, vr, do)
    np.testing.assert_allclose(dq, dq_m, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk, dk_m.reshape(B, Hkv, G, Tk, D).sum(axis=2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, dv_m.reshape(B, Hkv, G, Tk, D).sum(axis=2), rtol=0, atol=1e-12)


def test_gradients_scale_with_the_output_gradient():
    """The gradients are linear in dO: doubling dO (exact in bf16) doubles each of them."""
    q, k, v, do = inputs(1, 4, 2, 6, 6, 8, seed=99)
    g1 = bwd(q, k, v, do)
    g2 = bwd(q, k, v, gi.scale_pow2_bf16(do, 1))
    for a, c in zip(g1, g2):
        np.testing.assert_allclose(c, 2 * a, rtol=0, atol=1e-12)


def test_backward_rejects_what_the_forward_rejects():
    q, k, v, do = inputs(1, 4, 2, 5, 5, 8, seed=101)
    with pytest.raises(ValueError):
        bwd(q, k[:, :1], v[:, :1].copy(), do[:, :3].copy())   # shapes disagree
    with pytest.raises(ValueError):
        bwd(q, np.ascontiguousarray(k[:, :, :4]), np.ascontiguousarray(v[:, :, :4]), do)  # Tq > Tk
