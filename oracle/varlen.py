"""fp64 oracle for sequences of different lengths: packed, padded and paged forms.

TEST INFRASTRUCTURE ONLY, like the rest of this package: the tests, the smoke check
and the bench's CPU-baseline / reference arm may use it; the product never does.

What the forms mean. "注意力家族", section Mask 与增量位置, lists what a real attention
implementation must handle besides the causal mask: padding masks and packed
segments, and query lengths that differ from the cache length. It also says the mask
must be built from absolute positions / cache offsets, not from the tensors' shapes.
"Attention Architecture Evolution", section GDN, uses `cu_seqlens` as the boundaries
of packed sequences. Read plainly, a batch of sequences of different lengths is S
independent problems. Each one is the dense causal GQA of the o_a equation ("注意力家族",
section 统一记号) over its own rows: its L_q query rows sit at positions
L_k - L_q .. L_k - 1 of its own L_k keys, and a row sees no token of any other
sequence and no padding.

The oracle is that reading written out. It cuts each sequence out of the packed or
padded arrays and calls the fp64 row oracle (`gqa_oracle.c`) on it. Nothing is
tiled, fused or reordered.

Layouts (uint16 arrays of bf16 bits, D contiguous):
  packed (cu given):  x[H, rows, D]. Sequence s owns rows cu[s] .. cu[s+1]-1.
  padded (cu None):   x[S, H, rows, D]. Sequence s is batch s and owns rows
                      0 .. len[s]-1 (len None = all rows).
Queries and keys each pick their own form, so a packed chunk can attend over a
padded cache.

Paged caches are not on the pages. The plainest reading of a paged cache is a
lookup: logical position t of sequence b lives at row t % page of pool page
table[b, t // page]. `gather_pages` writes that lookup out, and the result feeds the
padded form.
"""
from __future__ import annotations

import numpy as np

from . import attention as _dense_attention


def _bounds(n_seq, cu, lens, rows, name):
    """(batch index, first row, length) of every sequence of one side."""
    out = []
    if cu is not None:
        cu = np.asarray(cu, dtype=np.int64).reshape(-1)
        if cu.size != n_seq + 1 or cu[0] < 0:
            raise ValueError(f"cu_{name} must have S + 1 entries starting at >= 0")
        for s in range(n_seq):
            start, end = int(cu[s]), int(cu[s + 1])
            if end < start or end > rows:
                raise ValueError(f"cu_{name} must be non-decreasing and within the rows")
            out.append((0, start, end - start))
    else:
        for s in range(n_seq):
            length = rows if lens is None else int(lens[s])
            if length < 0 or length > rows:
                raise ValueError(f"len_{name}[{s}] outside [0, rows]")
            out.append((s, 0, length))
    return out


def _plane(x, batch, start, length, packed):
    """[1, H, length, D] contiguous copy of one sequence's rows."""
    sl = x[:, start:start + length] if packed else x[batch, :, start:start + length]
    return np.ascontiguousarray(sl[None])


def attention_varlen(q, k, v, n_seq, cu_q=None, cu_k=None, len_q=None, len_k=None, scale=None,
                     window=0, with_lse=False, threads=None):
    """fp64 outputs of S independent causal GQA problems.

    q is packed [H_q, rows_q, D] if cu_q is given, else padded [S, H_q, rows_q, D];
    k and v likewise with cu_k / len_k. Returns an array in q's layout (float64),
    NaN on rows that belong to no sequence, and with ``with_lse`` the natural-log
    LSE laid out like q without D ([H_q, rows_q] or [S, H_q, rows_q]), NaN likewise.
    """
    packed_q, packed_k = cu_q is not None, cu_k is not None
    rows_q = q.shape[1] if packed_q else q.shape[2]
    rows_k = k.shape[1] if packed_k else k.shape[2]
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    bq = _bounds(n_seq, cu_q, len_q, rows_q, "q")
    bk = _bounds(n_seq, cu_k, len_k, rows_k, "k")
    out = np.full(q.shape, np.nan, dtype=np.float64)
    lse = np.full(q.shape[:-1], np.nan, dtype=np.float64) if with_lse else None
    for s in range(n_seq):
        (b_q, r_q, l_q), (b_k, r_k, l_k) = bq[s], bk[s]
        if l_q > l_k:
            raise ValueError(f"sequence {s}: more queries ({l_q}) than keys ({l_k})")
        if l_q == 0:
            continue
        qs = _plane(q, b_q, r_q, l_q, packed_q)
        ks = _plane(k, b_k, r_k, l_k, packed_k)
        vs = _plane(v, b_k, r_k, l_k, packed_k)
        res = _dense_attention(qs, ks, vs, scale=scale, threads=threads, with_lse=with_lse,
                               window=window)
        o_s, lse_s = (res[0][0], res[1][0]) if with_lse else (res[0], None)
        if packed_q:
            out[:, r_q:r_q + l_q] = o_s
            if with_lse:
                lse[:, r_q:r_q + l_q] = lse_s
        else:
            out[b_q, :, r_q:r_q + l_q] = o_s
            if with_lse:
                lse[b_q, :, r_q:r_q + l_q] = lse_s
    return (out, lse) if with_lse else out


def gather_pages(pool, block_table, lens, page, rows=None):
    """Contiguous [B, H, rows, D] cache from a paged pool [pages, H, page, D].

    Row t < lens[b] of batch b is row t % page of pool page block_table[b, t // page];
    rows at or past lens[b] are zero (never read by the attention above)."""
    lens = np.asarray(lens, dtype=np.int64)
    table = np.asarray(block_table, dtype=np.int64)
    B = lens.size
    H, D = pool.shape[1], pool.shape[3]
    rows = int(lens.max()) if rows is None else int(rows)
    out = np.zeros((B, H, rows, D), dtype=pool.dtype)
    for b in range(B):
        t = np.arange(int(lens[b]))
        out[b, :, t] = pool[table[b, t // page], :, t % page]
    return out
