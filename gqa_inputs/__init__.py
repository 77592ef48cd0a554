"""Seeded synthetic inputs shared by the fp64 oracle and the GPU harness.

This module holds the input recipe only: the workload shapes and a
counter-based N(0,1) -> bf16 generator (``gen.c``). It contains none of the
attention arithmetic, so both sides of every parity check can import it
without sharing any code of the method.

Tensors are returned as numpy ``uint16`` arrays of bf16 bit patterns in the
``[B, H, T, D]`` layout (D innermost) that the pages' interface uses
("注意力家族", section 最小语义实现: q is [B,H_q,T_q,D], k and v are
[B,H_kv,T_k,D]). Tensor ids: Q=0, K=1, V=2.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libgqa_inputs.so")

TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2
# streams of the integer draws: query-chunk lengths, cached-prefix lengths, page order
STREAM_LEN, STREAM_PREFIX, STREAM_PAGES = 3, 4, 5
TENSOR_DO = 6  # the output gradient dO of the backward pass, N(0,1) bf16 like Q/K/V


def build(force: bool = False) -> str:
    """Compile gen.c into libgqa_inputs.so next to it (gcc, -O3, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O3", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.gqa_gen_normal_bf16.restype = ctypes.c_int
        lib.gqa_gen_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64,
                                            ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int]
        lib.gqa_gen_key.restype = ctypes.c_uint64
        lib.gqa_gen_key.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
        lib.gqa_gen_words.restype = None
        lib.gqa_gen_words.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64,
                                      ctypes.c_uint64, ctypes.c_void_p]
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def normal_bf16(seed: int, tensor_id: int, shape, start: int = 0, threads: int | None = None,
                out: np.ndarray | None = None) -> np.ndarray:
    """Elements [start, start + prod(shape)) of stream (seed, tensor_id), as bf16 bits.

    ``out`` may be a preallocated C-contiguous uint16 array (for example a
    pinned host buffer viewed through numpy).
    """
    n = int(np.prod(shape, dtype=np.int64)) if len(shape) else 1
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags["C_CONTIGUOUS"] and out.size == n
    _load().gqa_gen_normal_bf16(int(seed), int(tensor_id), int(start), n,
                                out.ctypes.data, int(threads or default_threads()))
    return out


def words(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """Raw 64-bit words [start, start + n) of stream (seed, stream)."""
    out = np.empty(int(n), dtype=np.uint64)
    if n:
        _load().gqa_gen_words(int(seed), int(stream), int(start), int(n), out.ctypes.data)
    return out


def uniform_ints(seed: int, stream: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n integers in [lo, hi]: lo + word mod (hi - lo + 1) (int64)."""
    if hi < lo:
        raise ValueError("empty range")
    w = words(seed, stream, n)
    return (lo + (w % np.uint64(hi - lo + 1)).astype(np.int64)).astype(np.int64)


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    """A permutation of 0..n-1: the stable argsort of n words (int64)."""
    return np.argsort(words(seed, stream, n), kind="stable").astype(np.int64)


def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round-to-nearest-even), returning bit patterns.

    Used to build hand-written fixtures (values that are exact in bf16)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def scale_pow2_bf16(u16: np.ndarray, exponent: int) -> np.ndarray:
    """Multiply bf16 values by 2**exponent. Exact for normal values that stay normal."""
    f = bf16_bits_to_f32(u16) * np.float32(2.0 ** exponent)
    out = f32_to_bf16_bits(f)
    return out.reshape(np.shape(u16))


@dataclass(frozen=True)
class Workload:
    """Shape and recipe of one synthetic workload (seeded iid N(0,1) bf16)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Tq: int
    Tk: int
    D: int
    q_pow2: int = 0      # Q multiplied by 2**q_pow2 after bf16 rounding
    seed: int = 0
    window: int = 0      # sliding window (0 = plain causal); a mask setting, not data

    @property
    def q_shape(self):
        return (self.B, self.Hq, self.Tq, self.D)

    @property
    def kv_shape(self):
        return (self.B, self.Hkv, self.Tk, self.D)

    def make_dout(self, threads: int | None = None):
        """The output gradient dO for this workload's backward pass ([B, Hq, Tq, D] bf16 bits)."""
        return normal_bf16(self.seed, TENSOR_DO, self.q_shape, threads=threads)

    def make(self, threads: int | None = None, q_out=None, k_out=None, v_out=None):
        """Generate (q, k, v) bf16 bit arrays for this workload."""
        q = normal_bf16(self.seed, TENSOR_Q, self.q_shape, threads=threads, out=q_out)
        if self.q_pow2:
            q[...] = scale_pow2_bf16(q, self.q_pow2)
        k = normal_bf16(self.seed, TENSOR_K, self.kv_shape, threads=threads, out=k_out)
        v = normal_bf16(self.seed, TENSOR_V, self.kv_shape, threads=threads, out=v_out)
        return q, k, v


# The five workloads of the benchmark plan. Names state what each one is.
TINY = Workload("tiny causal GQA B2 Hq4 Hkv2 T128 D64", 2, 4, 2, 128, 128, 64)
GQA_PREFILL = Workload("GQA prefill B4 Hq32 Hkv8 T4096 D128", 4, 32, 8, 4096, 4096, 128)
MQA_LONG = Workload("MQA long prefill B1 Hq32 Hkv1 T32768 D128", 1, 32, 1, 32768, 32768, 128)
GQA_DECODE = Workload("GQA decode B64 Hq32 Hkv8 Tk32768 D128", 64, 32, 8, 1, 32768, 128)
MHA_SUFFIX = Workload("MHA suffix B8 H16 Tq512 at 7680 over Tk8192 D128 Qx4", 8, 16, 16, 512, 8192, 128,
                      q_pow2=2)

# Workloads of the extension rows (sliding window, short decode chunks).
SWA_PREFILL = Workload("GQA sliding-window prefill B4 Hq32 Hkv8 T4096 W1024 D128", 4, 32, 8, 4096, 4096,
                       128, window=1024)
CHUNK_DECODE = Workload("GQA verify chunk B64 Hq32 Hkv8 Tq4 Tk32768 D128", 64, 32, 8, 4, 32768, 128)

WORKLOADS = {
    "tiny": TINY,
    "gqa_prefill": GQA_PREFILL,
    "mqa_long": MQA_LONG,
    "gqa_decode": GQA_DECODE,
    "mha_suffix": MHA_SUFFIX,
    "swa_prefill": SWA_PREFILL,
    "chunk_decode": CHUNK_DECODE,
}


def cu_from_lengths(lengths) -> np.ndarray:
    """Sequence boundaries [0, l0, l0 + l1, ...] (int32) of packed sequences."""
    lengths = np.asarray(lengths, dtype=np.int64)
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


@dataclass(frozen=True)
class VarlenWorkload:
    """Packed sequences of a variable length (chunked prefill of a serving step).

    Sequence s has a new chunk of L_q(s) query tokens ~ U[q_lo, q_hi] after a cached
    prefix of P(s) ~ U[prefix_lo, prefix_hi] tokens, so it attends over
    L_k(s) = P(s) + L_q(s) keys. Q, K and V are token-major, [total, H, D] (the packed
    layout of serving engines); every value is iid N(0,1) bf16 from the same streams
    as the dense workloads."""
    name: str
    S: int
    Hq: int
    Hkv: int
    D: int
    q_lo: int
    q_hi: int
    prefix_lo: int = 0
    prefix_hi: int = 0
    seed: int = 0
    window: int = 0

    def lengths(self):
        lq = uniform_ints(self.seed, STREAM_LEN, self.S, self.q_lo, self.q_hi)
        if self.prefix_hi > 0:
            pre = uniform_ints(self.seed, STREAM_PREFIX, self.S, self.prefix_lo, self.prefix_hi)
        else:
            pre = np.zeros(self.S, dtype=np.int64)
        return lq, lq + pre

    def make(self, threads: int | None = None):
        """(q, k, v, cu_q, cu_k): token-major bf16 bit arrays and int32 boundaries."""
        lq, lk = self.lengths()
        cu_q, cu_k = cu_from_lengths(lq), cu_from_lengths(lk)
        q = normal_bf16(self.seed, TENSOR_Q, (int(cu_q[-1]), self.Hq, self.D), threads=threads)
        k = normal_bf16(self.seed, TENSOR_K, (int(cu_k[-1]), self.Hkv, self.D), threads=threads)
        v = normal_bf16(self.seed, TENSOR_V, (int(cu_k[-1]), self.Hkv, self.D), threads=threads)
        return q, k, v, cu_q, cu_k


@dataclass(frozen=True)
class PagedDecodeWorkload:
    """Decode over a paged KV cache with a per-sequence cache length.

    Sequence b has L(b) ~ U[len_lo, len_hi] cached tokens (its T_q new queries are the
    last T_q of them) held in ceil(L(b) / page) pages of `page` tokens. The pool holds
    exactly the pages in use, in a seeded random order (a fragmented cache), laid out
    [pages, page, H_kv, D] (token-major inside a page); block_table[b, i] is the pool
    page of the sequence's i-th page, -1 past its last page."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    len_lo: int
    len_hi: int
    page: int
    Tq: int = 1
    seed: int = 0
    window: int = 0

    def lengths(self):
        return uniform_ints(self.seed, STREAM_LEN, self.B, self.len_lo, self.len_hi)

    def make(self, threads: int | None = None):
        """(q, k_pool, v_pool, lengths, block_table)."""
        lens = self.lengths()
        n_pages = (lens + self.page - 1) // self.page
        total = int(n_pages.sum())
        order = permutation(self.seed, STREAM_PAGES, total)
        width = int(n_pages.max())
        table = np.full((self.B, width), -1, dtype=np.int32)
        at = 0
        for b in range(self.B):
            table[b, :n_pages[b]] = order[at:at + n_pages[b]]
            at += int(n_pages[b])
        q = normal_bf16(self.seed, TENSOR_Q, (self.B, self.Hq, self.Tq, self.D), threads=threads)
        k = normal_bf16(self.seed, TENSOR_K, (total, self.page, self.Hkv, self.D), threads=threads)
        v = normal_bf16(self.seed, TENSOR_V, (total, self.page, self.Hkv, self.D), threads=threads)
        return q, k, v, lens.astype(np.int32), table


# Workloads of the variable-length row.
VARLEN_PREFILL = VarlenWorkload("GQA packed varlen prefill S16 chunks U[256,8192] Hq32 Hkv8 D128",
                                16, 32, 8, 128, 256, 8192)
CHUNKED_PREFILL = VarlenWorkload("GQA chunked prefill S32 chunks U[128,2048] after prefixes U[0,8192] "
                                 "Hq32 Hkv8 D128", 32, 32, 8, 128, 128, 2048, 0, 8192)
PAGED_DECODE = PagedDecodeWorkload("GQA paged decode B64 Hq32 Hkv8 D128 lengths U[4096,32768] page 64",
                                   64, 32, 8, 128, 4096, 32768, 64)

VARLEN_WORKLOADS = {
    "varlen_prefill": VARLEN_PREFILL,
    "chunked_prefill": CHUNKED_PREFILL,
    "paged_decode": PAGED_DECODE,
}
