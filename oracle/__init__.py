"""fp64 CPU oracle for causal grouped-query softmax attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this package; the product
(``grouped_query_softmax_b200``) never does, and the two share no code.

The arithmetic lives in ``gqa_oracle.c`` (plain C, double precision, one
output row at a time, straight from the o_a definition of "注意力家族",
section 统一记号). This module only builds that file and marshals numpy
arrays of bf16 bit patterns into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_LIB = os.path.join(_HERE, "libgqa_oracle.so")


def build(force: bool = False) -> str:
    """Compile gqa_oracle.c into libgqa_oracle.so (gcc -O2, IEEE double, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _bind(lib):
    ll, vp, i32 = ctypes.c_longlong, ctypes.c_void_p, ctypes.c_int
    lib.gqa_oracle_rows.restype = i32
    lib.gqa_oracle_rows.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                    ll, ll, ll, ll, ll, ll, ctypes.c_double,
                                    vp, ll, vp, vp, i32]
    lib.gqa_oracle_rows_window.restype = i32
    lib.gqa_oracle_rows_window.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                           ll, ll, ll, ll, ll, ll, ctypes.c_double, i32,
                                           vp, ll, vp, vp, i32]
    lib.gqa_oracle_bwd.restype = i32
    lib.gqa_oracle_bwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                   ll, ll, ll, ll, ll, ll, ctypes.c_double, i32,
                                   vp, vp, vp, i32]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _plane_strides(arr: np.ndarray, name: str):
    """Element strides (batch, head) of a [B, H, T, D] uint16 array whose rows are packed."""
    if arr.dtype != np.uint16 or arr.ndim != 4:
        raise ValueError(f"{name} must be a 4-D uint16 array of bf16 bits")
    es = arr.itemsize
    D = arr.shape[3]
    if arr.strides[3] != es or arr.strides[2] != D * es:
        raise ValueError(f"{name}: rows must be contiguous with row stride D")
    return arr.strides[0] // es, arr.strides[1] // es


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, rows, Tk: int | None = None,
                   scale: float | None = None, threads: int | None = None, with_lse: bool = False,
                   lib=None, window: int = 0):
    """fp64 output rows of causal GQA attention.

    q: uint16 [B, H_q, T_q, D]; k, v: uint16 [B, H_kv, T_cap, D] (rows packed,
    batch/head strides free; only the first ``Tk`` positions are read, default
    T_cap). ``rows`` are flat ids (b*H_q + a)*T_q + i. ``window`` > 0 restricts each
    query to its ``window`` most recent positions. Returns a float64 [len(rows), D]
    array (and the natural-log LSE per row if ``with_lse``).
    """
    B, Hq, Tq, D = q.shape
    Bk, Hkv, Tcap, Dk = k.shape
    if v.shape != k.shape or Bk != B or Dk != D:
        raise ValueError("shape mismatch between q, k and v")
    Tk = Tcap if Tk is None else int(Tk)
    q_sb, q_sh = _plane_strides(q, "q")
    k_sb, k_sh = _plane_strides(k, "k")
    v_sb, v_sh = _plane_strides(v, "v")
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    out = np.empty((rows.size, D), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64) if with_lse else None
    rc = (lib or _load()).gqa_oracle_rows_window(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Hq, Hkv, Tq, Tk, D,
        q_sb, q_sh, k_sb, k_sh, v_sb, v_sh, float(scale) if scale else 0.0, int(window),
        rows.ctypes.data, rows.size, out.ctypes.data, lse.ctypes.data if with_lse else None,
        int(threads or default_threads()))
    if rc == 1:
        raise ValueError("oracle rejected the arguments (H_q % H_kv != 0, T_q > T_k, bad row id ...)")
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return (out, lse) if with_lse else out


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, Tk: int | None = None,
              scale: float | None = None, threads: int | None = None, with_lse: bool = False,
              lib=None, window: int = 0):
    """All output rows, shaped [B, H_q, T_q, D] (float64)."""
    B, Hq, Tq, D = q.shape
    res = attention_rows(q, k, v, np.arange(B * Hq * Tq), Tk=Tk, scale=scale, threads=threads,
                         with_lse=with_lse, lib=lib, window=window)
    if with_lse:
        return res[0].reshape(B, Hq, Tq, D), res[1].reshape(B, Hq, Tq)
    return res.reshape(B, Hq, Tq, D)


def load_variant(path: str):
    """Load another build of gqa_oracle.c (same C interface); pass it as ``lib=``.

    Used only by the pin tests, which compile copies of the oracle with a
    planted mistake and check that some pin catches each one."""
    return _bind(ctypes.CDLL(path))


def attention_bwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, dout: np.ndarray, Tk: int | None = None,
                  scale: float | None = None, window: int = 0, threads: int | None = None, lib=None):
    """fp64 gradients (dq, dk, dv) of causal GQA attention for the output gradient ``dout``.

    q and dout: uint16 [B, H_q, T_q, D] (the same layout); k, v: uint16 [B, H_kv, T_cap, D]
    with the first ``Tk`` rows used. Returns float64 dq [B, H_q, T_q, D] and dk, dv
    [B, H_kv, Tk, D]; a KV head's dk and dv sum over all the query heads that read it.
    """
    B, Hq, Tq, D = q.shape
    Hkv, Tcap = k.shape[1], k.shape[2]
    if dout.shape != q.shape or v.shape != k.shape or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("shape mismatch between q, k, v and dout")
    Tk = Tcap if Tk is None else int(Tk)
    q_sb, q_sh = _plane_strides(q, "q")
    d_sb, d_sh = _plane_strides(dout, "dout")
    if (d_sb, d_sh) != (q_sb, q_sh):
        raise ValueError("dout must have q's strides")
    k_sb, k_sh = _plane_strides(k, "k")
    v_sb, v_sh = _plane_strides(v, "v")
    dq = np.empty((B, Hq, Tq, D), dtype=np.float64)
    dk = np.empty((B, Hkv, Tk, D), dtype=np.float64)
    dv = np.empty((B, Hkv, Tk, D), dtype=np.float64)
    rc = (lib or _load()).gqa_oracle_bwd(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, B, Hq, Hkv, Tq, Tk, D,
        q_sb, q_sh, k_sb, k_sh, v_sb, v_sh, float(scale) if scale else 0.0, int(window),
        dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, int(threads or default_threads()))
    if rc == 1:
        raise ValueError("oracle rejected the arguments (H_q % H_kv != 0, T_q > T_k ...)")
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return dq, dk, dv
