"""Causal grouped-query softmax attention on B200 (sm_100a): Python binding of libgqa.

Every step of the computation runs in the CUDA kernels of ``libgqa.so``; this
module only marshals arguments across the C ABI declared in ``include/gqa.h``.
The functions named ``gqa_*`` mirror the C entry points one to one (device
pointers as integers, sizes, strides, a stream handle). ``attn_fwd`` and
``attn_decode`` are conveniences for torch tensors: they check dtype, device and
layout, allocate the outputs (and the decode workspace) with torch, and call the
same entry points. PyTorch supplies device memory and streams only.

There is no CPU fallback: importing this package fails loudly if the CUDA
library has not been built.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "GqaError", "gqa_attn_fwd", "gqa_attn_fwd_ex", "gqa_attn_fwd_split", "gqa_attn_fwd_split_workspace_bytes",
    "gqa_attn_decode", "gqa_attn_decode_workspace_bytes",
    "gqa_attn_decode_num_splits", "gqa_attn_decode_static", "gqa_attn_decode_ex",
    "gqa_attn_decode_ex_workspace_bytes", "gqa_attn_decode_ex_num_splits", "gqa_status_string", "gqa_get_device_error",
    "gqa_selftest_bounded_wait", "attn_fwd", "attn_decode", "library_path",
    "GqaLayout", "gqa_attn_fwd_varlen", "gqa_attn_fwd_varlen_workspace_bytes", "gqa_attn_decode_varlen",
    "gqa_attn_decode_varlen_workspace_bytes", "gqa_attn_decode_varlen_num_splits",
    "gqa_attn_bwd", "gqa_attn_bwd_workspace_bytes", "attn_bwd", "gqa_attn_fwd_varlen_paged",
    "attn_fwd_varlen", "attn_decode_varlen",
    "GQA_OK", "GQA_ERR_INVALID_ARGUMENT", "GQA_ERR_UNSUPPORTED", "GQA_ERR_WORKSPACE",
    "GQA_ERR_CUDA", "GQA_ERR_TIMEOUT",
]

GQA_OK = 0
GQA_ERR_INVALID_ARGUMENT = 1
GQA_ERR_UNSUPPORTED = 2
GQA_ERR_WORKSPACE = 3
GQA_ERR_CUDA = 4
GQA_ERR_TIMEOUT = 5

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgqa.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build the CUDA library first "
        "(python -c 'import __graft_entry__ as g; g.build()'). There is no CPU fallback.")

_lib = ctypes.CDLL(_LIB_PATH)

_vp, _i32, _ll, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t

_lib.gqa_attn_fwd.restype = _i32
_lib.gqa_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                              _ll, _ll, _ll, _ll, _f32, _vp]
_lib.gqa_attn_fwd_ex.restype = _i32
_lib.gqa_attn_fwd_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                 _ll, _ll, _ll, _ll, _f32, _i32, _vp]
_lib.gqa_attn_fwd_split_workspace_bytes.restype = _sz
_lib.gqa_attn_fwd_split_workspace_bytes.argtypes = [_i32] * 7
_lib.gqa_attn_fwd_split.restype = _i32
_lib.gqa_attn_fwd_split.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                    _ll, _ll, _ll, _ll, _f32, _i32, _vp, _sz, _vp]
_lib.gqa_attn_fwd_host_workspace_bytes.restype = _sz
_lib.gqa_attn_fwd_host_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32]
_lib.gqa_attn_fwd_host.restype = _i32
_lib.gqa_attn_fwd_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32,
                                   _vp, _sz, _vp]
_lib.gqa_attn_decode_workspace_bytes.restype = _sz
_lib.gqa_attn_decode_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32]
_lib.gqa_attn_decode_num_splits.restype = _i32
_lib.gqa_attn_decode_num_splits.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32]
_lib.gqa_attn_decode.restype = _i32
_lib.gqa_attn_decode.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                 _ll, _ll, _ll, _ll, _f32, _i32, _vp, _sz, _vp]
_lib.gqa_attn_decode_ex_workspace_bytes.restype = _sz
_lib.gqa_attn_decode_ex_workspace_bytes.argtypes = [_i32] * 8
_lib.gqa_attn_decode_ex_num_splits.restype = _i32
_lib.gqa_attn_decode_ex_num_splits.argtypes = [_i32] * 8
_lib.gqa_attn_decode_ex.restype = _i32
_lib.gqa_attn_decode_ex.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                    _ll, _ll, _ll, _ll, _f32, _i32, _i32, _vp, _sz, _vp]
_lib.gqa_attn_decode_static.restype = _i32
_lib.gqa_attn_decode_static.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                        _ll, _ll, _ll, _ll, _f32, _i32, _vp]


class GqaLayout(ctypes.Structure):
    """C ``gqa_layout``: element strides (batch, head, row) of a bf16 operand; d is contiguous."""
    _fields_ = [("sb", _ll), ("sh", _ll), ("st", _ll)]


_lay = ctypes.POINTER(GqaLayout)
_lib.gqa_attn_fwd_varlen_workspace_bytes.restype = _sz
_lib.gqa_attn_fwd_varlen_workspace_bytes.argtypes = [_i32] * 4
_lib.gqa_attn_fwd_varlen.restype = _i32
_lib.gqa_attn_fwd_varlen.argtypes = ([_vp] * 9 + [_i32] * 7 + [_lay] * 4 + [_f32, _i32, _vp, _sz, _vp])
_lib.gqa_attn_fwd_varlen_paged.restype = _i32
_lib.gqa_attn_fwd_varlen_paged.argtypes = ([_vp] * 9 + [_i32] * 9 + [_lay] * 4 + [_f32, _i32, _vp, _sz, _vp])
_lib.gqa_attn_decode_varlen_workspace_bytes.restype = _sz
_lib.gqa_attn_decode_varlen_workspace_bytes.argtypes = [_i32] * 8
_lib.gqa_attn_decode_varlen_num_splits.restype = _i32
_lib.gqa_attn_decode_varlen_num_splits.argtypes = [_i32] * 8
_lib.gqa_attn_decode_varlen.restype = _i32
_lib.gqa_attn_decode_varlen.argtypes = ([_vp] * 6 + [_i32] * 9 + [_lay] * 2 + [_f32, _i32, _i32, _vp, _sz, _vp])
_lib.gqa_attn_bwd_workspace_bytes.restype = _sz
_lib.gqa_attn_bwd_workspace_bytes.argtypes = [_i32] * 6
_lib.gqa_attn_bwd.restype = _i32
_lib.gqa_attn_bwd.argtypes = [_vp] * 9 + [_i32] * 6 + [_ll] * 4 + [_f32, _i32, _vp, _sz, _vp]
_lib.gqa_status_string.restype = ctypes.c_char_p
_lib.gqa_status_string.argtypes = [_i32]
_lib.gqa_get_device_error.restype = _i32
_lib.gqa_get_device_error.argtypes = [_vp]
_lib.gqa_selftest_bounded_wait.restype = _i32
_lib.gqa_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, _vp]


def library_path() -> str:
    return _LIB_PATH


class GqaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {gqa_status_string(status)}" if what else gqa_status_string(status))


# ---------------------------------------------------------------- raw C entry points
def gqa_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                 softmax_scale=0.0, stream=None) -> int:
    """C ``gqa_attn_fwd``; pointers are integers (device addresses). Returns the status."""
    return _lib.gqa_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                             float(softmax_scale), stream)


def gqa_attn_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                    softmax_scale=0.0, window=0, stream=None) -> int:
    """C ``gqa_attn_fwd_ex``: ``gqa_attn_fwd`` with a sliding window (0 = causal only)."""
    return _lib.gqa_attn_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                                float(softmax_scale), int(window), stream)


def gqa_attn_fwd_split_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, window=0) -> int:
    """C ``gqa_attn_fwd_split_workspace_bytes`` (0: the launch does not split)."""
    return _lib.gqa_attn_fwd_split_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, window)


def gqa_attn_fwd_split(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                       softmax_scale=0.0, window=0, workspace=None, workspace_bytes=0, stream=None) -> int:
    """C ``gqa_attn_fwd_split``: ``gqa_attn_fwd_ex`` that may split the keys of the last wave's
    units over several CTAs (partials merged by log-sum-exp in a workspace). Returns the status."""
    return _lib.gqa_attn_fwd_split(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                                   float(softmax_scale), window, workspace, workspace_bytes, stream)


def gqa_attn_fwd_host_workspace_bytes(B, Hq, Hkv, Tq, Tk, D) -> int:
    return int(_lib.gqa_attn_fwd_host_workspace_bytes(B, Hq, Hkv, Tq, Tk, D))


def gqa_attn_fwd_host(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, softmax_scale=0.0, window=0,
                      workspace=None, workspace_bytes=0, stream=None) -> int:
    """C ``gqa_attn_fwd_host``: q, k, v, o, lse are HOST addresses; workspace a device address."""
    return _lib.gqa_attn_fwd_host(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, float(softmax_scale), int(window),
                                  workspace, workspace_bytes, stream)


def gqa_attn_decode_workspace_bytes(B, Hq, Hkv, Tk, D, num_splits=0) -> int:
    return int(_lib.gqa_attn_decode_workspace_bytes(B, Hq, Hkv, Tk, D, num_splits))


def gqa_attn_decode_num_splits(B, Hq, Hkv, Tk, D, num_splits=0) -> int:
    return int(_lib.gqa_attn_decode_num_splits(B, Hq, Hkv, Tk, D, num_splits))


def gqa_attn_decode(q, k_cache, v_cache, o, B, Hq, Hkv, Tk, D, k_sb, k_sh, v_sb, v_sh,
                    softmax_scale=0.0, num_splits=0, workspace=None, workspace_bytes=0,
                    stream=None) -> int:
    """C ``gqa_attn_decode``; pointers are integers (device addresses). Returns the status."""
    return _lib.gqa_attn_decode(q, k_cache, v_cache, o, B, Hq, Hkv, Tk, D, k_sb, k_sh, v_sb, v_sh,
                                float(softmax_scale), num_splits, workspace, workspace_bytes, stream)


def gqa_attn_decode_ex_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, window=0, num_splits=0) -> int:
    return int(_lib.gqa_attn_decode_ex_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, window, num_splits))


def gqa_attn_decode_ex_num_splits(B, Hq, Hkv, Tq, Tk, D, window=0, num_splits=0) -> int:
    return int(_lib.gqa_attn_decode_ex_num_splits(B, Hq, Hkv, Tq, Tk, D, window, num_splits))


def gqa_attn_decode_ex(q, k_cache, v_cache, o, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                       softmax_scale=0.0, window=0, num_splits=0, workspace=None, workspace_bytes=0,
                       stream=None) -> int:
    """C ``gqa_attn_decode_ex``: decode of 1 <= Tq <= 16 new queries per head, optional window."""
    return _lib.gqa_attn_decode_ex(q, k_cache, v_cache, o, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb,
                                   v_sh, float(softmax_scale), int(window), int(num_splits), workspace,
                                   workspace_bytes, stream)


def gqa_attn_decode_static(q, k_cache, v_cache, o, B, Hq, Hkv, Tk, D, k_sb, k_sh, v_sb, v_sh,
                           softmax_scale=0.0, num_splits=0, stream=None) -> int:
    """C ``gqa_attn_decode_static``: decode with the library's fixed 16 MiB device scratch
    instead of a caller workspace, for callers that cannot allocate device memory."""
    return _lib.gqa_attn_decode_static(q, k_cache, v_cache, o, B, Hq, Hkv, Tk, D, k_sb, k_sh, v_sb,
                                       v_sh, float(softmax_scale), num_splits, stream)


def _layout(x):
    if isinstance(x, GqaLayout):
        return x
    sb, sh, st = x
    return GqaLayout(int(sb), int(sh), int(st))


def gqa_attn_fwd_varlen_workspace_bytes(S, Hq, Hkv, max_seqlen_q) -> int:
    return int(_lib.gqa_attn_fwd_varlen_workspace_bytes(S, Hq, Hkv, max_seqlen_q))


def gqa_attn_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, seqlens_q, seqlens_k, S, Hq, Hkv,
                        D, rows_q, rows_k, max_seqlen_q, q_layout, k_layout, v_layout, o_layout,
                        softmax_scale=0.0, window=0, workspace=None, workspace_bytes=0,
                        stream=None) -> int:
    """C ``gqa_attn_fwd_varlen``; layouts are GqaLayout or (sb, sh, st) tuples in elements."""
    lq, lk, lv, lo = (_layout(x) for x in (q_layout, k_layout, v_layout, o_layout))
    return _lib.gqa_attn_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, seqlens_q, seqlens_k,
                                    S, Hq, Hkv, D, rows_q, rows_k, max_seqlen_q, ctypes.byref(lq),
                                    ctypes.byref(lk), ctypes.byref(lv), ctypes.byref(lo),
                                    float(softmax_scale), int(window), workspace, workspace_bytes, stream)


def gqa_attn_fwd_varlen_paged(q, k_pool, v_pool, o, lse, cu_seqlens_q, seqlens_q, seqlens_k, block_table,
                              page_size, num_pages, max_pages, S, Hq, Hkv, D, rows_q, max_seqlen_q, q_layout,
                              k_layout, v_layout, o_layout, softmax_scale=0.0, window=0, workspace=None,
                              workspace_bytes=0, stream=None) -> int:
    """C ``gqa_attn_fwd_varlen_paged``: variable-length forward over a paged key/value cache."""
    lq, lk, lv, lo = (_layout(x) for x in (q_layout, k_layout, v_layout, o_layout))
    return _lib.gqa_attn_fwd_varlen_paged(q, k_pool, v_pool, o, lse, cu_seqlens_q, seqlens_q, seqlens_k,
                                          block_table, page_size, num_pages, max_pages, S, Hq, Hkv, D, rows_q,
                                          max_seqlen_q, ctypes.byref(lq), ctypes.byref(lk), ctypes.byref(lv),
                                          ctypes.byref(lo), float(softmax_scale), int(window), workspace,
                                          workspace_bytes, stream)


def gqa_attn_decode_varlen_workspace_bytes(B, Hq, Hkv, Tq, max_seqlen_k, D, window=0, num_splits=0) -> int:
    return int(_lib.gqa_attn_decode_varlen_workspace_bytes(B, Hq, Hkv, Tq, max_seqlen_k, D, window, num_splits))


def gqa_attn_decode_varlen_num_splits(B, Hq, Hkv, Tq, max_seqlen_k, D, window=0, num_splits=0) -> int:
    return int(_lib.gqa_attn_decode_varlen_num_splits(B, Hq, Hkv, Tq, max_seqlen_k, D, window, num_splits))


def gqa_attn_decode_varlen(q, k_cache, v_cache, o, seqlens_k, block_table, page_size, num_pages,
                           max_pages, B, Hq, Hkv, Tq, max_seqlen_k, D, k_layout, v_layout,
                           softmax_scale=0.0, window=0, num_splits=0, workspace=None, workspace_bytes=0,
                           stream=None) -> int:
    """C ``gqa_attn_decode_varlen``: decode over per-sequence cache lengths, contiguous or paged."""
    lk, lv = _layout(k_layout), _layout(v_layout)
    return _lib.gqa_attn_decode_varlen(q, k_cache, v_cache, o, seqlens_k, block_table, page_size,
                                       num_pages, max_pages, B, Hq, Hkv, Tq, max_seqlen_k, D,
                                       ctypes.byref(lk), ctypes.byref(lv), float(softmax_scale),
                                       int(window), int(num_splits), workspace, workspace_bytes, stream)


def gqa_attn_bwd_workspace_bytes(B, Hq, Hkv, Tq, Tk, D) -> int:
    return int(_lib.gqa_attn_bwd_workspace_bytes(B, Hq, Hkv, Tq, Tk, D))


def gqa_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                 softmax_scale=0.0, window=0, workspace=None, workspace_bytes=0, stream=None) -> int:
    """C ``gqa_attn_bwd``: dq, dk, dv of the causal GQA forward for the output gradient dout."""
    return _lib.gqa_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                             float(softmax_scale), int(window), workspace, workspace_bytes, stream)


def gqa_status_string(status: int) -> str:
    return _lib.gqa_status_string(int(status)).decode()


def gqa_get_device_error(stream=None) -> int:
    return _lib.gqa_get_device_error(stream)


def gqa_selftest_bounded_wait(timeout_ns: int, stream=None) -> int:
    return _lib.gqa_selftest_bounded_wait(int(timeout_ns), stream)


# ---------------------------------------------------------------- torch conveniences
def _torch():
    import torch
    return torch


def _stream_handle(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check_bf16_cuda(t, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a bf16 CUDA tensor")


def _plane_strides(t, name):
    """(batch, head) element strides of a [B, H, T, D] tensor with packed rows."""
    if t.dim() != 4 or t.stride(3) != 1 or (t.size(2) > 1 and t.stride(2) != t.size(3)):
        raise ValueError(f"{name} must be [B, H, T, D] with rows packed (stride(3)=1, stride(2)=D)")
    return t.stride(0), t.stride(1)


def attn_fwd(q, k, v, *, Tk=None, scale=None, window=0, return_lse=False, out=None, stream=None, split=True,
             workspace=None):
    """o = causal GQA attention of q [B,Hq,Tq,D] over k, v [B,Hkv,T_cap,D] (first Tk rows).

    Query row i sits at position Tk - Tq + i; ``window`` > 0 limits it to its
    ``window`` most recent positions. Returns o (bf16, [B,Hq,Tq,D]) and, if
    ``return_lse``, the fp32 natural-log log-sum-exp [B,Hq,Tq].

    With ``split`` (the default) the call goes through gqa_attn_fwd_split, which may
    split the keys of the last wave's units over several CTAs (the results then agree with
    ``split=False``, gqa_attn_fwd_ex, within rounding rather than bit for bit);
    ``workspace`` is then a uint8 CUDA tensor of at least
    gqa_attn_fwd_split_workspace_bytes(...) bytes, allocated here when omitted.
    """
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_bf16_cuda(t, n)
    if not q.is_contiguous():
        raise ValueError("q must be contiguous [B, Hq, Tq, D]")
    B, Hq, Tq, D = q.shape
    Hkv = k.shape[1]
    Tk = k.shape[2] if Tk is None else int(Tk)
    if k.shape[0] != B or v.shape[:2] != k.shape[:2] or k.shape[3] != D or v.shape[3] != D:
        raise ValueError("q, k, v shapes disagree")
    if Tk > k.shape[2] or Tk > v.shape[2]:
        raise ValueError("Tk exceeds the cache capacity")
    k_sb, k_sh = _plane_strides(k, "k")
    v_sb, v_sh = _plane_strides(v, "v")
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device) if return_lse else None
    lse_ptr = lse.data_ptr() if lse is not None else None
    if not split:
        st = gqa_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr, B, Hq, Hkv, Tq, Tk,
                             D, k_sb, k_sh, v_sb, v_sh, float(scale or 0.0), int(window), _stream_handle(stream))
        if st != GQA_OK:
            raise GqaError(st, "gqa_attn_fwd_ex")
        return (out, lse) if return_lse else out
    need = gqa_attn_fwd_split_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, int(window))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if (need and workspace is not None) else None
    ws_bytes = workspace.numel() * workspace.element_size() if (need and workspace is not None) else 0
    st = gqa_attn_fwd_split(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr, B, Hq, Hkv, Tq, Tk, D,
                            k_sb, k_sh, v_sb, v_sh, float(scale or 0.0), int(window), ws_ptr, ws_bytes,
                            _stream_handle(stream))
    if st != GQA_OK:
        raise GqaError(st, "gqa_attn_fwd_split")
    return (out, lse) if return_lse else out


def attn_fwd_host(q, k, v, *, scale=None, window=0, return_lse=False, out=None, workspace=None, device=None,
                  stream=None, synchronize=True):
    """attn_fwd for operands in host memory: q [B,Hq,Tq,D] and k, v [B,Hkv,Tk,D], contiguous
    bf16 CPU tensors (pinned, for the copies to overlap the kernels). The library streams
    query-row chunks through a device workspace (gqa_attn_fwd_host) and writes o (and the
    fp32 LSE) into CPU tensors. With ``synchronize=False`` the call returns once the work is
    enqueued on ``stream``, and the outputs are valid once the stream reaches that point."""
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous bf16 CPU tensor")
    B, Hq, Tq, D = q.shape
    Hkv, Tk = k.shape[1], k.shape[2]
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("q, k, v shapes disagree")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=q.is_pinned())
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 CPU tensor shaped like q")
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, pin_memory=q.is_pinned()) if return_lse else None
    need = gqa_attn_fwd_host_workspace_bytes(B, Hq, Hkv, Tq, Tk, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8,
                                device=device if device is not None else torch.cuda.current_device())
    st = gqa_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                           lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Tq, Tk, D,
                           float(scale or 0.0), int(window), workspace.data_ptr(),
                           workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != GQA_OK:
        raise GqaError(st, "gqa_attn_fwd_host")
    if synchronize:
        if stream is None:
            torch.cuda.current_stream().synchronize()
        elif hasattr(stream, "synchronize"):
            stream.synchronize()
        else:
            torch.cuda.synchronize()
    return (out, lse) if return_lse else out


def attn_decode(q, k_cache, v_cache, *, Tk=None, scale=None, window=0, num_splits=0, out=None,
                workspace=None, stream=None):
    """One decode step: q [B,Hq,Tq,D] (Tq <= 16; or [B,Hq,D] for Tq = 1) over the first Tk
    cached keys; query row i sits at position Tk - Tq + i."""
    torch = _torch()
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check_bf16_cuda(t, n)
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    B, Hq, D = q.shape[0], q.shape[1], q.shape[-1]
    Tq = q.shape[2] if q.dim() == 4 else 1
    if q.numel() != B * Hq * Tq * D:
        raise ValueError("q must be [B, Hq, Tq, D] or [B, Hq, D]")
    Hkv = k_cache.shape[1]
    Tk = k_cache.shape[2] if Tk is None else int(Tk)
    k_sb, k_sh = _plane_strides(k_cache, "k_cache")
    v_sb, v_sh = _plane_strides(v_cache, "v_cache")
    if out is None:
        out = torch.empty_like(q)
    need = gqa_attn_decode_ex_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, window, num_splits)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = gqa_attn_decode_ex(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                            B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh, float(scale or 0.0),
                            int(window), int(num_splits), ws_ptr, ws_bytes, _stream_handle(stream))
    if st != GQA_OK:
        raise GqaError(st, "gqa_attn_decode_ex")
    return out


def _side_layout(t, name):
    """(packed?, rows, H, layout) of a varlen operand: packed [rows, H, D] or padded [S, H, rows, D]."""
    if t.stride(-1) != 1:
        raise ValueError(f"{name}: the last (D) axis must be contiguous")
    if t.dim() == 3:
        return True, t.shape[0], t.shape[1], (0, t.stride(1), t.stride(0))
    if t.dim() == 4:
        return False, t.shape[2], t.shape[1], (t.stride(0), t.stride(1), t.stride(2))
    raise ValueError(f"{name} must be packed [rows, H, D] or padded [S, H, rows, D]")


def _ptr(t):
    return t.data_ptr() if t is not None else None


def _int32_cuda(t, name):
    torch = _torch()
    if t is None:
        return None
    if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous int32 CUDA tensor")
    return t


def attn_fwd_varlen(q, k, v, *, cu_seqlens_q=None, cu_seqlens_k=None, seqlens_q=None, seqlens_k=None,
                    max_seqlen_q=None, scale=None, window=0, return_lse=False, out=None, workspace=None,
                    block_table=None, pool_layout="NHD", stream=None):
    """S independent causal GQA problems of different lengths in one call.

    Each side is packed, a 3-D [rows, H, D] tensor (any row/head strides, so token-major
    [total, H, D] and a transposed head-major buffer both work) with int32 boundaries
    ``cu_seqlens_*`` [S + 1], or padded, a 4-D [S, H, rows, D] tensor with optional
    lengths ``seqlens_*`` [S]. Sequence s's L_q query rows sit at positions L_k - L_q ..
    L_k - 1 of its own keys. Returns o shaped like q (rows of no sequence untouched)
    and, with ``return_lse``, the fp32 LSE [Hq, rows_q] (packed) or [S, Hq, rows_q].

    With ``block_table`` (int32 [S, max_pages]) the keys are paged: k and v are pools
    [pages, page, Hkv, D] ("NHD") or [pages, Hkv, page, D] ("HND") and ``seqlens_k`` gives
    each sequence's key count.
    """
    if block_table is not None:
        return _attn_fwd_varlen_paged(q, k, v, cu_seqlens_q, seqlens_q, seqlens_k, block_table, max_seqlen_q,
                                      scale, window, return_lse, out, workspace, pool_layout, stream)
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_bf16_cuda(t, n)
    cu_q, cu_k = _int32_cuda(cu_seqlens_q, "cu_seqlens_q"), _int32_cuda(cu_seqlens_k, "cu_seqlens_k")
    len_q, len_k = _int32_cuda(seqlens_q, "seqlens_q"), _int32_cuda(seqlens_k, "seqlens_k")
    packed_q, rows_q, Hq, lay_q = _side_layout(q, "q")
    packed_k, rows_k, Hkv, lay_k = _side_layout(k, "k")
    _, _, _, lay_v = _side_layout(v, "v")
    if packed_q != (cu_q is not None) or packed_k != (cu_k is not None):
        raise ValueError("a packed (3-D) side needs cu_seqlens; a padded (4-D) side must not have it")
    if v.shape != k.shape or q.shape[-1] != k.shape[-1]:
        raise ValueError("q, k, v shapes disagree")
    D = q.shape[-1]
    S = cu_q.numel() - 1 if packed_q else q.shape[0]
    S_k = cu_k.numel() - 1 if packed_k else k.shape[0]
    if S != S_k or S <= 0:
        raise ValueError("queries and keys describe different numbers of sequences")
    if max_seqlen_q is None:  # convenience: one device-to-host read
        if packed_q:
            max_seqlen_q = int((cu_q[1:] - cu_q[:-1]).max().item())
        else:
            max_seqlen_q = int(len_q.max().item()) if len_q is not None else rows_q
    max_seqlen_q = max(1, int(max_seqlen_q))
    if out is None:
        out = torch.empty_like(q)
    _, _, _, lay_o = _side_layout(out, "out")
    lse = None
    if return_lse:
        lse = torch.empty(((Hq, rows_q) if packed_q else (S, Hq, rows_q)), dtype=torch.float32,
                          device=q.device)
    need = gqa_attn_fwd_varlen_workspace_bytes(S, Hq, Hkv, max_seqlen_q)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = gqa_attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse),
                             _ptr(cu_q), _ptr(cu_k), _ptr(len_q), _ptr(len_k), S, Hq, Hkv, D, rows_q,
                             rows_k, max_seqlen_q, lay_q, lay_k, lay_v, lay_o, float(scale or 0.0),
                             int(window), workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    if st != GQA_OK:
        raise GqaError(st, "gqa_attn_fwd_varlen")
    return (out, lse) if return_lse else out


def attn_decode_varlen(q, k_cache, v_cache, seqlens_k, *, block_table=None, max_seqlen_k=None,
                       pool_layout="NHD", scale=None, window=0, num_splits=0, out=None, workspace=None,
                       stream=None):
    """Decode of q [B, Hq, Tq, D] (Tq <= 16; or [B, Hq, D]) over per-sequence cache lengths.

    Contiguous cache (``block_table`` None): k_cache/v_cache [B, Hkv, T_cap, D] with any
    batch/head/row strides. Paged cache: a pool [pages, page, Hkv, D] ("NHD") or
    [pages, Hkv, page, D] ("HND") and an int32 block table [B, max_pages]. Sequence b's
    queries are the last Tq of its seqlens_k[b] positions.
    """
    torch = _torch()
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check_bf16_cuda(t, n)
    seqlens_k = _int32_cuda(seqlens_k, "seqlens_k")
    table = _int32_cuda(block_table, "block_table")
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    B, Hq, D = q.shape[0], q.shape[1], q.shape[-1]
    Tq = q.shape[2] if q.dim() == 4 else 1
    if seqlens_k is None or seqlens_k.numel() != B:
        raise ValueError("seqlens_k must hold one length per sequence")
    if k_cache.shape != v_cache.shape or k_cache.dim() != 4 or k_cache.stride(3) != 1:
        raise ValueError("k_cache and v_cache must be 4-D with a contiguous D axis and equal shapes")

    def lay(t):
        if table is None:
            return (t.stride(0), t.stride(1), t.stride(2))
        if pool_layout == "NHD":
            return (t.stride(0), t.stride(2), t.stride(1))
        if pool_layout == "HND":
            return (t.stride(0), t.stride(1), t.stride(2))
        raise ValueError("pool_layout must be 'NHD' or 'HND'")

    if table is None:
        Hkv = k_cache.shape[1]
        page_size = num_pages = max_pages = 0
        cap = k_cache.shape[2]
        max_seqlen_k = cap if max_seqlen_k is None else int(max_seqlen_k)
        if max_seqlen_k > cap:
            raise ValueError("max_seqlen_k exceeds the cache rows")
    else:
        Hkv = k_cache.shape[2] if pool_layout == "NHD" else k_cache.shape[1]
        page_size = k_cache.shape[1] if pool_layout == "NHD" else k_cache.shape[2]
        num_pages = k_cache.shape[0]
        if table.dim() != 2 or table.shape[0] != B:
            raise ValueError("block_table must be [B, max_pages]")
        max_pages = table.shape[1]
        max_seqlen_k = max_pages * page_size if max_seqlen_k is None else int(max_seqlen_k)
    if out is None:
        out = torch.empty_like(q)
    need = gqa_attn_decode_varlen_workspace_bytes(B, Hq, Hkv, Tq, max_seqlen_k, D, window, num_splits)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = gqa_attn_decode_varlen(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                                seqlens_k.data_ptr(), _ptr(table), page_size, num_pages, max_pages, B, Hq,
                                Hkv, Tq, max_seqlen_k, D, lay(k_cache), lay(v_cache), float(scale or 0.0),
                                int(window), int(num_splits), _ptr(workspace),
                                workspace.numel() if workspace is not None else 0, _stream_handle(stream))
    if st != GQA_OK:
        raise GqaError(st, "gqa_attn_decode_varlen")
    return out


def attn_bwd(q, k, v, o, dout, lse, *, Tk=None, scale=None, window=0, dq=None, dk=None, dv=None,
             workspace=None, stream=None):
    """Gradients (dq, dk, dv) of ``attn_fwd(q, k, v)`` for the output gradient ``dout``.

    o and lse are the forward's output and its log-sum-exp (``attn_fwd(..., return_lse=True)``);
    q, o, dout [B,Hq,Tq,D] contiguous; k, v [B,Hkv,T_cap,D] (first Tk rows). dk and dv are
    [B,Hkv,Tk,D]; a KV head's gradient sums over the query heads that read it.
    """
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _check_bf16_cuda(t, n)
    for t, n in ((q, "q"), (o, "o"), (dout, "dout")):
        if not t.is_contiguous() or t.shape != q.shape:
            raise ValueError(f"{n} must be contiguous and shaped like q")
    if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise TypeError("lse must be a contiguous fp32 CUDA tensor")
    B, Hq, Tq, D = q.shape
    Hkv = k.shape[1]
    Tk = k.shape[2] if Tk is None else int(Tk)
    k_sb, k_sh = _plane_strides(k, "k")
    v_sb, v_sh = _plane_strides(v, "v")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty((B, Hkv, Tk, D), dtype=q.dtype, device=q.device) if dk is None else dk
    dv = torch.empty((B, Hkv, Tk, D), dtype=q.dtype, device=q.device) if dv is None else dv
    need = gqa_attn_bwd_workspace_bytes(B, Hq, Hkv, Tq, Tk, D)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = gqa_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                      dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                      float(scale or 0.0), int(window), workspace.data_ptr(), workspace.numel(),
                      _stream_handle(stream))
    if st != GQA_OK:
        raise GqaError(st, "gqa_attn_bwd")
    return dq, dk, dv


def _attn_fwd_varlen_paged(q, k_pool, v_pool, cu_seqlens_q, seqlens_q, seqlens_k, block_table, max_seqlen_q,
                           scale, window, return_lse, out, workspace, pool_layout, stream):
    torch = _torch()
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _check_bf16_cuda(t, n)
    cu_q = _int32_cuda(cu_seqlens_q, "cu_seqlens_q")
    len_q, len_k = _int32_cuda(seqlens_q, "seqlens_q"), _int32_cuda(seqlens_k, "seqlens_k")
    table = _int32_cuda(block_table, "block_table")
    if len_k is None:
        raise ValueError("a paged cache needs seqlens_k")
    packed_q, rows_q, Hq, lay_q = _side_layout(q, "q")
    if packed_q != (cu_q is not None):
        raise ValueError("packed (3-D) queries need cu_seqlens_q; padded (4-D) queries must not have it")
    if k_pool.shape != v_pool.shape or k_pool.dim() != 4 or k_pool.stride(3) != 1:
        raise ValueError("k_pool and v_pool must be 4-D with a contiguous D axis and equal shapes")
    if pool_layout == "NHD":
        num_pages, page, Hkv, D = k_pool.shape
        lay = lambda t: (t.stride(0), t.stride(2), t.stride(1))
    elif pool_layout == "HND":
        num_pages, Hkv, page, D = k_pool.shape
        lay = lambda t: (t.stride(0), t.stride(1), t.stride(2))
    else:
        raise ValueError("pool_layout must be 'NHD' or 'HND'")
    S = cu_q.numel() - 1 if packed_q else q.shape[0]
    if table.dim() != 2 or table.shape[0] != S or len_k.numel() != S:
        raise ValueError("block_table must be [S, max_pages] and seqlens_k [S]")
    if max_seqlen_q is None:
        if packed_q:
            max_seqlen_q = int((cu_q[1:] - cu_q[:-1]).max().item())
        else:
            max_seqlen_q = int(len_q.max().item()) if len_q is not None else rows_q
    max_seqlen_q = max(1, int(max_seqlen_q))
    if out is None:
        out = torch.empty_like(q)
    _, _, _, lay_o = _side_layout(out, "out")
    lse = None
    if return_lse:
        lse = torch.empty(((Hq, rows_q) if packed_q else (S, Hq, rows_q)), dtype=torch.float32, device=q.device)
    need = gqa_attn_fwd_varlen_workspace_bytes(S, Hq, Hkv, max_seqlen_q)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = gqa_attn_fwd_varlen_paged(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), out.data_ptr(), _ptr(lse),
                                   _ptr(cu_q), _ptr(len_q), len_k.data_ptr(), table.data_ptr(), page, num_pages,
                                   table.shape[1], S, Hq, Hkv, D, rows_q, max_seqlen_q, lay_q, lay(k_pool),
                                   lay(v_pool), lay_o, float(scale or 0.0), int(window), workspace.data_ptr(),
                                   workspace.numel(), _stream_handle(stream))
    if st != GQA_OK:
        raise GqaError(st, "gqa_attn_fwd_varlen_paged")
    return (out, lse) if return_lse else out
