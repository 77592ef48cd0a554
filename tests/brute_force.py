"""A second, independent fp64 formulation used only to pin the oracle on tiny inputs.

It follows the pages' matrix form rather than the oracle's row loop: expand
K/V to one plane per query head with a repeat along the head axis
("注意力家族", section 最小语义实现, the repeat_interleave step), build the full
T_q x T_k score matrix, add an explicit mask matrix built from absolute
query/key positions (same section, query_pos / key_pos), softmax along keys,
then one matrix product with V. Every step is a numpy array operation on whole
matrices, so a slip in the oracle's indices shows up as a mismatch here.
"""
import numpy as np


def brute_force_attention(qf: np.ndarray, kf: np.ndarray, vf: np.ndarray, scale=None, window=0):
    """qf [B,Hq,Tq,D], kf/vf [B,Hkv,Tk,D], float64 values. Returns [B,Hq,Tq,D].

    window > 0 adds the sliding-window mask: keys more than window-1 positions
    before the query are hidden too."""
    B, Hq, Tq, D = qf.shape
    Hkv, Tk = kf.shape[1], kf.shape[2]
    assert Hq % Hkv == 0 and Tq <= Tk
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    rep = Hq // Hkv
    k_exp = np.repeat(kf, rep, axis=1)  # heads k0,k0,..,k1,k1,.. (interleaved repeat)
    v_exp = np.repeat(vf, rep, axis=1)
    scores = np.matmul(qf, np.swapaxes(k_exp, -1, -2)) * scale  # [B,Hq,Tq,Tk]
    query_pos = np.arange(Tk - Tq, Tk)[:, None]
    key_pos = np.arange(Tk)[None, :]
    hidden = key_pos > query_pos
    if window > 0:
        hidden = hidden | (key_pos <= query_pos - window)
    mask = np.where(hidden, -np.inf, 0.0)  # [Tq,Tk]
    scores = scores + mask
    scores = scores - scores.max(axis=-1, keepdims=True)
    w = np.exp(scores)
    w = w / w.sum(axis=-1, keepdims=True)
    return np.matmul(w, v_exp)
