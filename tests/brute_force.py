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


def brute_force_segments(qf, kf, vf, seg_q, pos_q, seg_k, pos_k, scale=None, window=0):
    """Matrix form over flattened token axes, with an explicit segment mask.

    qf [Hq, Nq, D], kf/vf [Hkv, Nk, D] (float64); seg_* / pos_* give every query row
    and key row its sequence id (-1 = belongs to none) and its absolute position in
    that sequence. Key j is visible to row i iff both are in the same sequence,
    pos_k[j] <= pos_q[i] and, with a window, pos_k[j] > pos_q[i] - window. One
    Nq x Nk score matrix per head, softmax over keys, one product with V. Rows that
    see no key come out NaN."""
    Hq, Nq, D = qf.shape
    Hkv = kf.shape[0]
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    rep = Hq // Hkv
    k_exp = np.repeat(kf, rep, axis=0)
    v_exp = np.repeat(vf, rep, axis=0)
    seg_q, pos_q = np.asarray(seg_q)[:, None], np.asarray(pos_q)[:, None]
    seg_k, pos_k = np.asarray(seg_k)[None, :], np.asarray(pos_k)[None, :]
    visible = (seg_q == seg_k) & (seg_q >= 0) & (pos_k <= pos_q)
    if window > 0:
        visible &= pos_k > pos_q - window
    scores = np.matmul(qf, np.swapaxes(k_exp, -1, -2)) * scale
    scores = np.where(visible[None], scores, -np.inf)
    with np.errstate(invalid="ignore"):
        scores = scores - scores.max(axis=-1, keepdims=True)
        w = np.exp(scores)
        w = w / w.sum(axis=-1, keepdims=True)
    return np.matmul(w, v_exp)
