#!/usr/bin/env python
"""Benchmark of causal grouped-query softmax attention on B200.

One step = one pass of the hot path over one batch of synthetic input:
  * headline: gqa_attn_fwd on the GQA prefill workload (B4 Hq32 Hkv8 T4096 D128),
    metric TFLOP/s with FLOPs = 4 * D * Hq * B * (causal-visible query/key pairs);
  * "decode" object: gqa_attn_decode on the GQA decode workload (B64 Hq32 Hkv8,
    T_k 32768, D128), metric KV GB/s = (K + V bytes) / time.
Inputs are seeded iid N(0,1) rounded to bf16 (see gqa_inputs), resident in HBM
when the timed region starts. Under torchrun every rank runs its own copy of the
workload (independent problems, no data-path collective): weak scaling, value =
all ranks' work / max-over-ranks time.

--impl reference times the fp64 CPU oracle (the only other implementation of the
method here) on a bounded row sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import gqa_inputs as gi  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
_CSRC = "grouped_query_softmax_b200/csrc/"
# The sources each kernel is compiled from: a traffic figure stays valid while these hash
# to the value recorded with it.
KERNEL_SOURCES = {
    "gqa_fwd_sm100_kernel": [_CSRC + "fwd_sm100.cuh", _CSRC + "sm100_ptx.cuh"],
    "gqa_decode_sm100_kernel": [_CSRC + "decode_sm100.cuh", _CSRC + "sm100_ptx.cuh"],
    "gqa_bwd_sm100_kernel": [_CSRC + "bwd_sm100.cuh", _CSRC + "sm100_ptx.cuh", _CSRC + "gqa_internal.h"],
}
KERNEL_SOURCES["gqa_fwd_sm100_kernel_varlen"] = KERNEL_SOURCES["gqa_fwd_sm100_kernel"]
KERNEL_SOURCES["gqa_decode_sm100_kernel_varlen"] = KERNEL_SOURCES["gqa_decode_sm100_kernel"]


# ---------------------------------------------------------------- work counts
def visible_pairs(Tq: int, Tk: int, window: int = 0) -> int:
    """Visible (query, key) pairs per (b, a): row i sees Tk - Tq + i + 1 keys, at most
    `window` of them inside a sliding window."""
    if window <= 0:
        return Tq * (Tk - Tq) + Tq * (Tq + 1) // 2
    seen = np.minimum(np.arange(Tk - Tq, Tk, dtype=np.int64) + 1, window)
    return int(seen.sum())


def algorithmic_flops(w) -> float:
    return 4.0 * w.D * w.Hq * w.B * visible_pairs(w.Tq, w.Tk, w.window)


def kv_bytes(w) -> int:
    return 2 * w.B * w.Hkv * w.Tk * w.D * 2


def qo_bytes(w) -> int:
    return 2 * w.B * w.Hq * w.Tq * w.D * 2


def row_flops(w, rows) -> float:
    i = np.asarray(rows) % w.Tq
    seen = w.Tk - w.Tq + i + 1
    if w.window > 0:
        seen = np.minimum(seen, w.window)
    return float(np.sum(4.0 * w.D * seen))


def is_decode(w) -> bool:
    """Workloads of a few new queries over a long cache run through gqa_attn_decode_ex."""
    return w.Tq <= 16 and w.Tk >= 1024


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()[:16]


def tensor_peak(peaks, peak_src, clocks):
    """(peak, description): the sustained GEMM figure when the timed region ran at the power
    cap, otherwise the burst figure."""
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    burst = peaks["bf16_tflops"]
    if capped:
        return (peaks.get("bf16_tflops_sustained", burst),
                f"{peak_src} bf16_tflops_sustained (sw_power_cap active in the timed region)")
    return burst, f"{peak_src} bf16_tflops (burst; kernel timed alone)"


def tensor_roofline(achieved, peaks, peak_src, clocks, traffic, kernel):
    """The roofline object of a tensor-bound row: the power-cap-aware peak and the fraction
    of it, with the fractions of the burst and sustained figures for context."""
    peak, src = tensor_peak(peaks, peak_src, clocks)
    burst = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained", burst)
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic, "peak_source": src,
            "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
            "frac_of_spec_2250": achieved / 2250.0, "kernel": kernel}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel sources still
    match the ones that capture was taken with; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("kernel_source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the GPU is busy."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.samples = []
        self.proc = None
        self.gpu_id = gpu_id

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.gpu_id is not None:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        threading.Thread(target=self._reader, daemon=True).start()

    def _reader(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        window = [s for t, s in self.samples if t0 <= t <= t1]
        scope = "timed region"
        if len(window) < 3:
            window = [s for _, s in self.samples]
            scope = "whole run (timed region shorter than the sampling interval)"
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "scope": "unavailable"}
        sm = [num(s[1]) for s in window if num(s[1]) is not None]
        smax = [num(s[2]) for s in window if num(s[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in window for i in range(4) if s[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(window), "scope": scope}


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- GPU measurements
def to_device(arr_u16, dev):
    import torch
    return torch.from_numpy(arr_u16.view(np.int16)).to(dev).view(torch.bfloat16)


def timed(fn, steps, warmup, world, dev):
    """Run fn() warmup times, then time exactly `steps` calls on the current stream.
    Returns (max-over-ranks ms for the whole timed region, t_start, t_end wall)."""
    import torch
    for _ in range(warmup):
        fn()
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    ms = start.elapsed_time(end)
    return max_over_ranks(ms, world, dev), t0, t1


def measure_prefill(w, steps, warmup, world, dev, e2e_steps):
    import torch
    import grouped_query_softmax_b200 as gqa
    q, k, v = w.make()
    qd, kd, vd = to_device(q, dev), to_device(k, dev), to_device(v, dev)
    od = torch.empty_like(qd)
    fn = lambda: gqa.attn_fwd(qd, kd, vd, out=od, window=w.window)
    ms, t0, t1 = timed(fn, steps, warmup, world, dev)
    st = gqa.gqa_get_device_error(torch.cuda.current_stream().cuda_stream)
    if st != gqa.GQA_OK:
        raise RuntimeError(f"device error after prefill timing: {gqa.gqa_status_string(st)}")
    res = {"ms_total": ms, "t0": t0, "t1": t1, "launches": steps}

    # end to end through the public host-memory call (gqa_attn_fwd_host): pinned host inputs
    # in, host output out, every step; its device workspace is allocated once, outside
    del qd, kd, vd, od
    torch.cuda.empty_cache()
    qh = torch.from_numpy(q.view(np.int16)).pin_memory().view(torch.bfloat16)
    kh = torch.from_numpy(k.view(np.int16)).pin_memory().view(torch.bfloat16)
    vh = torch.from_numpy(v.view(np.int16)).pin_memory().view(torch.bfloat16)
    oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(gqa.gqa_attn_fwd_host_workspace_bytes(w.B, w.Hq, w.Hkv, w.Tq, w.Tk, w.D), dtype=torch.uint8,
                     device=dev)

    def e2e_step():
        gqa.attn_fwd_host(qh, kh, vh, out=oh, window=w.window, workspace=ws, synchronize=False)
    e2e_ms, _, _ = timed(e2e_step, e2e_steps, 1, world, dev)
    res["e2e_ms_total"] = e2e_ms
    res["e2e_steps"] = e2e_steps
    res["h2d_bytes"] = int(q.nbytes + k.nbytes + v.nbytes)
    res["d2h_bytes"] = int(q.nbytes)
    del ws
    return res


def measure_decode(w, steps, warmup, world, dev, e2e_steps):
    import torch
    import grouped_query_softmax_b200 as gqa
    q, k, v = w.make()
    qd, kd, vd = to_device(q, dev), to_device(k, dev), to_device(v, dev)
    od = torch.empty_like(qd)
    splits = gqa.gqa_attn_decode_ex_num_splits(w.B, w.Hq, w.Hkv, w.Tq, w.Tk, w.D, w.window, 0)
    need = gqa.gqa_attn_decode_ex_workspace_bytes(w.B, w.Hq, w.Hkv, w.Tq, w.Tk, w.D, w.window, 0)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    fn = lambda: gqa.attn_decode(qd, kd, vd, out=od, workspace=ws, window=w.window)
    ms, t0, t1 = timed(fn, steps, warmup, world, dev)
    st = gqa.gqa_get_device_error(torch.cuda.current_stream().cuda_stream)
    if st != gqa.GQA_OK:
        raise RuntimeError(f"device error after decode timing: {gqa.gqa_status_string(st)}")
    res = {"ms_total": ms, "t0": t0, "t1": t1, "splits": splits,
           "launches": steps * (1 if splits == 1 else 2)}
    qh = torch.from_numpy(q.view(np.int16)).pin_memory()
    kh = torch.from_numpy(k.view(np.int16)).pin_memory()
    vh = torch.from_numpy(v.view(np.int16)).pin_memory()
    oh = torch.empty(q.shape, dtype=torch.int16).pin_memory()
    qi, ki, vi, oi = (x.view(torch.int16) for x in (qd, kd, vd, od))

    def e2e_step():
        qi.copy_(qh, non_blocking=True)
        ki.copy_(kh, non_blocking=True)
        vi.copy_(vh, non_blocking=True)
        gqa.attn_decode(qd, kd, vd, out=od, workspace=ws, window=w.window)
        oh.copy_(oi, non_blocking=True)
    e2e_ms, _, _ = timed(e2e_step, e2e_steps, 1, world, dev)
    res.update(e2e_ms_total=e2e_ms, e2e_steps=e2e_steps, h2d_bytes=int(q.nbytes + k.nbytes + v.nbytes),
               d2h_bytes=int(q.nbytes))
    del qd, kd, vd, od, ws
    torch.cuda.empty_cache()
    return res


def bwd_flops(w) -> float:
    """Backward FLOPs: five products per visible pair (S recomputed, dP, dV, dK, dQ), each
    2 * D per pair and query head: 10 * D * Hq * B * pairs = 2.5x the forward's."""
    return 10.0 * w.D * w.Hq * w.B * visible_pairs(w.Tq, w.Tk, w.window)


def measure_bwd(w, steps, warmup, world, dev):
    """gqa_attn_bwd on a dense workload: prep + attention backward + dQ rounding per step;
    the forward's output and log-sum-exp are computed once, before the timed region."""
    import torch
    import grouped_query_softmax_b200 as gqa
    q, k, v = w.make()
    do = w.make_dout()
    qd, kd, vd, dod = (to_device(x, dev) for x in (q, k, v, do))
    o, lse = gqa.attn_fwd(qd, kd, vd, return_lse=True)
    dq = torch.empty_like(qd)
    dk = torch.empty_like(kd)
    dv = torch.empty_like(vd)
    ws = torch.empty(gqa.gqa_attn_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.Tq, w.Tk, w.D), dtype=torch.uint8,
                     device=dev)
    fn = lambda: gqa.attn_bwd(qd, kd, vd, o, dod, lse, dq=dq, dk=dk, dv=dv, workspace=ws)
    ms, t0, t1 = timed(fn, steps, warmup, world, dev)
    st = gqa.gqa_get_device_error(torch.cuda.current_stream().cuda_stream)
    if st != gqa.GQA_OK:
        raise RuntimeError(f"device error after backward timing: {gqa.gqa_status_string(st)}")
    del qd, kd, vd, dod, o, lse, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return {"ms_total": ms, "t0": t0, "t1": t1, "launches": 3 * steps}


def varlen_flops(w) -> float:
    """4 * D * Hq * sum over sequences of their causal-visible pairs."""
    lq, lk = w.lengths()
    return 4.0 * w.D * w.Hq * sum(visible_pairs(int(a), int(b), w.window) for a, b in zip(lq, lk) if a)


def measure_paged_prefill(w, page, steps, warmup, world, dev):
    """The chunked-prefill workload with each sequence's keys in a paged pool (pages of
    `page` keys in a seeded random order, [pages, page, Hkv, D])."""
    import torch
    import grouped_query_softmax_b200 as gqa
    q, k, v, cu_q, cu_k = w.make()
    lq, lk = w.lengths()
    n_pages = (lk + page - 1) // page
    order = gi.permutation(w.seed, gi.STREAM_PAGES, int(n_pages.sum()))
    pool_k = np.zeros((order.size, page, w.Hkv, w.D), dtype=np.uint16)
    pool_v = np.zeros_like(pool_k)
    table = np.full((w.S, int(n_pages.max())), -1, dtype=np.int32)
    at = 0
    for s in range(w.S):
        for i in range(int(n_pages[s])):
            pg = order[at]
            at += 1
            table[s, i] = pg
            r0, r1 = int(cu_k[s]) + i * page, int(cu_k[s]) + min((i + 1) * page, int(lk[s]))
            pool_k[pg, :r1 - r0] = k[r0:r1]
            pool_v[pg, :r1 - r0] = v[r0:r1]
    qd, kd, vd = to_device(q, dev), to_device(pool_k, dev), to_device(pool_v, dev)
    cq = torch.tensor(cu_q, device=dev)
    ld = torch.tensor(lk.astype(np.int32), device=dev)
    td = torch.tensor(table, device=dev)
    od = torch.empty_like(qd)
    max_q = int(lq.max())
    ws = torch.empty(gqa.gqa_attn_fwd_varlen_workspace_bytes(w.S, w.Hq, w.Hkv, max_q), dtype=torch.uint8, device=dev)
    fn = lambda: gqa.attn_fwd_varlen(qd, kd, vd, cu_seqlens_q=cq, seqlens_k=ld, block_table=td, max_seqlen_q=max_q,
                                     window=w.window, out=od, workspace=ws)
    ms, _, _ = timed(fn, steps, warmup, world, dev)
    st = gqa.gqa_get_device_error(torch.cuda.current_stream().cuda_stream)
    if st != gqa.GQA_OK:
        raise RuntimeError(f"device error after paged prefill timing: {gqa.gqa_status_string(st)}")
    del qd, kd, vd, od, ws
    torch.cuda.empty_cache()
    return {"ms_total": ms, "launches": 2 * steps}


def paged_kv_bytes(w) -> int:
    """K + V bytes of every cached key, read once per KV head."""
    return 2 * int(w.lengths().sum()) * w.Hkv * w.D * 2


def measure_varlen(w, steps, warmup, world, dev, e2e_steps=0):
    """gqa_attn_fwd_varlen on a packed workload (plan kernel + attention kernel per step)."""
    import torch
    import grouped_query_softmax_b200 as gqa
    q, k, v, cu_q, cu_k = w.make()
    lq, _ = w.lengths()
    qd, kd, vd = to_device(q, dev), to_device(k, dev), to_device(v, dev)
    cq = torch.tensor(cu_q, device=dev)
    ck = torch.tensor(cu_k, device=dev)
    od = torch.empty_like(qd)
    max_q = int(lq.max())
    ws = torch.empty(gqa.gqa_attn_fwd_varlen_workspace_bytes(w.S, w.Hq, w.Hkv, max_q), dtype=torch.uint8,
                     device=dev)
    fn = lambda: gqa.attn_fwd_varlen(qd, kd, vd, cu_seqlens_q=cq, cu_seqlens_k=ck, max_seqlen_q=max_q,
                                     window=w.window, out=od, workspace=ws)
    ms, t0, t1 = timed(fn, steps, warmup, world, dev)
    st = gqa.gqa_get_device_error(torch.cuda.current_stream().cuda_stream)
    if st != gqa.GQA_OK:
        raise RuntimeError(f"device error after varlen timing: {gqa.gqa_status_string(st)}")
    res = {"ms_total": ms, "t0": t0, "t1": t1, "launches": 2 * steps, "tokens_q": int(cu_q[-1]),
           "tokens_k": int(cu_k[-1])}
    if e2e_steps:
        hosts = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in (q, k, v)]
        devs = [x.view(torch.int16) for x in (qd, kd, vd)]
        oh = torch.empty(q.shape, dtype=torch.int16).pin_memory()

        def e2e_step():
            for d_, h_ in zip(devs, hosts):
                d_.copy_(h_, non_blocking=True)
            fn()
            oh.copy_(od.view(torch.int16), non_blocking=True)
        e2e_ms, _, _ = timed(e2e_step, e2e_steps, 1, world, dev)
        res.update(e2e_ms_total=e2e_ms, e2e_steps=e2e_steps, h2d_bytes=int(q.nbytes + k.nbytes + v.nbytes),
                   d2h_bytes=int(q.nbytes))
    del qd, kd, vd, od, ws
    torch.cuda.empty_cache()
    return res


def measure_paged_decode(w, steps, warmup, world, dev, e2e_steps=0):
    """gqa_attn_decode_varlen over the paged pool of a PagedDecodeWorkload."""
    import torch
    import grouped_query_softmax_b200 as gqa
    q, kp, vp, lens, table = w.make()
    qd, kd, vd = to_device(q, dev), to_device(kp, dev), to_device(vp, dev)
    ld = torch.tensor(lens, device=dev)
    td = torch.tensor(table, device=dev)
    od = torch.empty_like(qd)
    max_k = int(lens.max())
    need = gqa.gqa_attn_decode_varlen_workspace_bytes(w.B, w.Hq, w.Hkv, w.Tq, max_k, w.D, w.window, 0)
    splits = gqa.gqa_attn_decode_varlen_num_splits(w.B, w.Hq, w.Hkv, w.Tq, max_k, w.D, w.window, 0)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    fn = lambda: gqa.attn_decode_varlen(qd, kd, vd, ld, block_table=td, max_seqlen_k=max_k, window=w.window,
                                        out=od, workspace=ws)
    ms, t0, t1 = timed(fn, steps, warmup, world, dev)
    st = gqa.gqa_get_device_error(torch.cuda.current_stream().cuda_stream)
    if st != gqa.GQA_OK:
        raise RuntimeError(f"device error after paged decode timing: {gqa.gqa_status_string(st)}")
    res = {"ms_total": ms, "t0": t0, "t1": t1, "splits": splits,
           "launches": steps * (1 if splits == 1 else 2)}
    if e2e_steps:
        hosts = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in (q, kp, vp)]
        devs = [x.view(torch.int16) for x in (qd, kd, vd)]
        oh = torch.empty(q.shape, dtype=torch.int16).pin_memory()

        def e2e_step():
            for d_, h_ in zip(devs, hosts):
                d_.copy_(h_, non_blocking=True)
            fn()
            oh.copy_(od.view(torch.int16), non_blocking=True)
        e2e_ms, _, _ = timed(e2e_step, e2e_steps, 1, world, dev)
        res.update(e2e_ms_total=e2e_ms, e2e_steps=e2e_steps, h2d_bytes=int(q.nbytes + kp.nbytes + vp.nbytes),
                   d2h_bytes=int(q.nbytes))
    del qd, kd, vd, od, ws
    torch.cuda.empty_cache()
    return res


def varlen_config(w):
    c = {"workload": w.name, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
         "q_len": f"U[{w.q_lo},{w.q_hi}]", "seed": w.seed, "causal": True, "layout": "token-major packed"}
    if w.prefix_hi:
        c["cached_prefix"] = f"U[{w.prefix_lo},{w.prefix_hi}]"
    return c


# ---------------------------------------------------------------- the oracle on the host
def oracle_sample(w, budget_s: float, threads: int, q=None, k=None, v=None):
    """Time the fp64 oracle on a seeded row sample sized to about budget_s seconds.
    Returns (flops_done, seconds, rows)."""
    import oracle
    if q is None:
        q, k, v = w.make()
    rng = np.random.default_rng(0)
    total = w.B * w.Hq * w.Tq
    # calibrate the parallel rate on a probe of several rows per thread
    probe = rng.integers(0, total, size=min(total, 8 * threads))
    t = time.perf_counter()
    oracle.attention_rows(q, k, v, probe, threads=threads, window=w.window)
    dt = max(time.perf_counter() - t, 1e-6)
    rate = row_flops(w, probe) / dt
    mean_row = 4.0 * w.D * visible_pairs(w.Tq, w.Tk, w.window) / w.Tq
    n = int(min(total, max(8 * threads, budget_s * rate / mean_row)))
    for _ in range(3):
        rows = np.sort(rng.choice(total, size=n, replace=False)) if n < total else np.arange(total)
        t = time.perf_counter()
        oracle.attention_rows(q, k, v, rows, threads=threads, window=w.window)
        dt = time.perf_counter() - t
        if dt >= 0.5 * budget_s or n >= total:
            break
        # the probe under-estimated the parallel rate: resize from the measured run
        n = int(min(total, n * budget_s / max(dt, 1e-3)))
    return row_flops(w, rows), dt, rows


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------- main
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gqa_prefill", choices=sorted(gi.WORKLOADS) + sorted(gi.VARLEN_WORKLOADS),
                    help="main workload (a varlen or paged one is measured alone, e.g. for profiling)")
    ap.add_argument("--decode-workload", default="gqa_decode", choices=sorted(gi.WORKLOADS))
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    ap.add_argument("--no-extensions", action="store_true",
                    help="skip the sliding-window, decode-chunk and variable-length measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--backward", action="store_true",
                    help="measure only the backward pass of the main (dense) workload, e.g. for profiling")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the main workload's batch size / sequence count (for profiling a smaller case)")
    return ap.parse_args(argv)


def workload_config(w, extra=None):
    c = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Tq": w.Tq, "Tk": w.Tk, "D": w.D,
         "q_scale": 2 ** w.q_pow2, "seed": w.seed, "causal": True}
    if w.window:
        c["window"] = w.window
    if extra:
        c.update(extra)
    return c


def metric_of(w):
    if is_decode(w):
        return "GQA attn KV GB/s (decode) on 1 B200, % of roofline", "GB/s"
    return "GQA attn TFLOP/s (prefill) on 1 B200, % of roofline", "TFLOP/s"


def throughput(w, ms_per_step, world):
    if is_decode(w):
        return world * kv_bytes(w) / (ms_per_step * 1e-3) / 1e9
    return world * algorithmic_flops(w) / (ms_per_step * 1e-3) / 1e12


def reference_arm(args, rank, world):
    """The oracle as the reference arm: rank 0 alone runs it; other ranks exit 0."""
    if rank != 0:
        return
    if args.workload not in gi.WORKLOADS:
        raise SystemExit("--impl reference times the oracle on the dense workloads only")
    w = gi.WORKLOADS[args.workload]
    threads = cpu_threads()
    q, k, v = w.make()
    per_step_budget = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, per_step_budget, threads, q, k, v)
    flops = secs = 0.0
    rows_total = 0
    for _ in range(args.steps):
        f, s, rows = oracle_sample(w, per_step_budget, threads, q, k, v)
        flops += f
        secs += s
        rows_total += len(rows)
    metric, unit = metric_of(w)
    if is_decode(w):
        frac = rows_total / (args.steps * w.B * w.Hq * w.Tq)
        value = frac * kv_bytes(w) * args.steps / secs / 1e9
    else:
        value = flops / secs / 1e12
    sample = f"{rows_total} output rows in {args.steps} steps (row-sampled, fp64, {per_step_budget:.1f} s per step)"
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def backward_main(args, rank, world, local, dev, peaks, peak_src, w):
    """The backward pass of a dense workload as the main line (profiling and focused runs)."""
    sampler = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[local])
    sampler.start()
    time.sleep(0.2)
    r = measure_bwd(w, args.steps, args.warmup, world, dev)
    ms_step = r["ms_total"] / args.steps
    achieved = bwd_flops(w) / (ms_step * 1e-3) / 1e12
    clocks = sampler.summary(r["t0"], r["t1"])
    sampler.stop()
    line = {"metric": "GQA attn backward TFLOP/s on 1 B200, % of roofline", "value": world * achieved,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, {"pass": "backward (dQ, dK, dV)", "l2": "inputs larger than L2 (no flush)",
                                          "parallelism": f"dp{world} (independent problems per rank)"}),
            "roofline": tensor_roofline(achieved, peaks, peak_src, clocks,
                                        load_traffic("gqa_bwd_sm100_kernel", w.name),
                                        "gqa_bwd_prep_kernel + gqa_bwd_sm100_kernel + gqa_bwd_dq_kernel"),
            "gpu_launches": r["launches"], "clocks": clocks}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def varlen_main(args, rank, world, local, dev, peaks, peak_src):
    """A variable-length or paged workload as the main line (profiling and focused runs)."""
    import dataclasses
    w = gi.VARLEN_WORKLOADS[args.workload]
    if args.batch > 0:
        field = "B" if isinstance(w, gi.PagedDecodeWorkload) else "S"
        w = dataclasses.replace(w, **{field: args.batch}, name=f"{w.name} ({field} {args.batch})")
    sampler = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[local])
    sampler.start()
    time.sleep(0.2)
    if isinstance(w, gi.PagedDecodeWorkload):
        r = measure_paged_decode(w, args.steps, args.warmup, world, dev, args.e2e_steps)
        work, unit, scale = paged_kv_bytes(w), "GB/s", 1e9
        metric = "GQA paged decode KV GB/s on 1 B200, % of roofline"
        config = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "Tq": w.Tq,
                  "cache_len": f"U[{w.len_lo},{w.len_hi}]", "page": w.page, "splits": r["splits"]}
        peak, bound, src = peaks["hbm_gbs"], "hbm", f"{peak_src} hbm_gbs (copy, read+write bytes)"
        kernel = "gqa_decode_sm100_kernel<varlen> + gqa_decode_combine_kernel"
    else:
        r = measure_varlen(w, args.steps, args.warmup, world, dev, args.e2e_steps)
        work, unit, scale = varlen_flops(w), "TFLOP/s", 1e12
        metric = "GQA varlen prefill TFLOP/s on 1 B200, % of roofline"
        config = varlen_config(w) | {"tokens_q": r["tokens_q"], "tokens_k": r["tokens_k"]}
        peak, bound, src = None, "tensor", None  # tensor_roofline below chooses the peak
        kernel = "gqa_varlen_plan_kernel + gqa_fwd_sm100_kernel<varlen>"
    ms_step = r["ms_total"] / args.steps
    achieved = work / (ms_step * 1e-3) / scale
    clocks = sampler.summary(r["t0"], r["t1"])
    sampler.stop()
    if bound == "tensor":
        roof = tensor_roofline(achieved, peaks, peak_src, clocks,
                               load_traffic("gqa_fwd_sm100_kernel_varlen", w.name), kernel)
    else:
        roof = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": load_traffic("gqa_decode_sm100_kernel_varlen", w.name), "peak_source": src,
                "kernel": kernel}
    line = {"metric": metric, "value": world * achieved, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config | {"l2": "inputs larger than L2 (no flush)",
                                "parallelism": f"dp{world} (independent problems per rank)"},
            "roofline": roof,
            "gpu_launches": r["launches"], "clocks": clocks}
    if args.e2e_steps:
        e2e_ms = r["e2e_ms_total"] / r["e2e_steps"]
        line["e2e"] = {"value": world * work / (e2e_ms * 1e-3) / scale, "unit": unit,
                       "h2d_bytes_per_step": r["h2d_bytes"], "d2h_bytes_per_step": r["d2h_bytes"],
                       "ms_per_step": e2e_ms, "steps": r["e2e_steps"]}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus > 1 needs torchrun (one process per GPU)")
    if args.impl == "reference":
        return reference_arm(args, rank, world)

    import torch
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    import grouped_query_softmax_b200 as gqa  # noqa: F401  (fails loudly without libgqa.so)

    peaks, peak_src = load_peaks()
    if args.workload in gi.VARLEN_WORKLOADS:
        return varlen_main(args, rank, world, local, dev, peaks, peak_src)
    w = gi.WORKLOADS[args.workload]
    if args.batch > 0:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch, name=f"{w.name} (batch {args.batch})")
    if args.backward:
        return backward_main(args, rank, world, local, dev, peaks, peak_src, w)
    gpu_id = None
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        gpu_id = vis.split(",")[local]
    elif world > 1:
        gpu_id = str(local)
    sampler = ClockSampler(gpu_id if gpu_id is not None else "0")
    sampler.start()
    time.sleep(0.2)

    metric, unit = metric_of(w)
    if is_decode(w):
        r = measure_decode(w, args.steps, args.warmup, world, dev, args.e2e_steps)
    else:
        r = measure_prefill(w, args.steps, args.warmup, world, dev, args.e2e_steps)
    ms_step = r["ms_total"] / args.steps
    value = throughput(w, ms_step, world)
    e2e_ms = r["e2e_ms_total"] / r["e2e_steps"]
    clocks = sampler.summary(r["t0"], r["t1"])

    if is_decode(w):
        per_launch_bytes = kv_bytes(w) + qo_bytes(w)
        achieved = per_launch_bytes / (ms_step * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": load_traffic("gqa_decode_sm100_kernel", w.name),
                "peak_source": f"{peak_src} hbm_gbs (copy, read+write bytes)",
                "kernel": "gqa_decode_sm100_kernel + gqa_decode_combine_kernel (one call per step)"}
    else:
        achieved = algorithmic_flops(w) / (ms_step * 1e-3) / 1e12
        roof = tensor_roofline(achieved, peaks, peak_src, clocks,
                               load_traffic("gqa_fwd_sm100_kernel", w.name), "gqa_fwd_sm100_kernel")

    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, {"l2": "inputs larger than L2 (no flush)",
                                          "parallelism": f"dp{world} (independent problems per rank)"}),
            "roofline": roof,
            "e2e": {"value": throughput(w, e2e_ms, world), "unit": unit,
                    "h2d_bytes_per_step": r["h2d_bytes"], "d2h_bytes_per_step": r["d2h_bytes"],
                    "ms_per_step": e2e_ms, "steps": r["e2e_steps"],
                    "call": ("gqa_attn_decode_ex after host-to-device copies of q, k, v" if is_decode(w) else
                             "gqa_attn_fwd_host: pinned host q, k, v, o; query-row chunks overlap copies "
                             "and kernels")},
            "gpu_launches": r["launches"], "clocks": clocks}

    if not args.no_decode and not is_decode(w):
        wd = gi.WORKLOADS[args.decode_workload]
        rd = measure_decode(wd, max(3, args.steps // 20), max(3, args.warmup), world, dev,
                            max(2, args.e2e_steps // 5))
        msd = rd["ms_total"] / max(3, args.steps // 20)
        gbs = throughput(wd, msd, world)
        ach = (kv_bytes(wd) + qo_bytes(wd)) / (msd * 1e-3) / 1e9
        line["decode"] = {
            "metric": "KV GB/s", "value": gbs, "unit": "GB/s", "ms_per_step": msd,
            "steps": max(3, args.steps // 20), "config": workload_config(wd, {"splits": rd["splits"]}),
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"],
                         "traffic": load_traffic("gqa_decode_sm100_kernel", wd.name),
                         "peak_source": f"{peak_src} hbm_gbs (copy, read+write bytes)"},
            "e2e": {"value": throughput(wd, rd["e2e_ms_total"] / rd["e2e_steps"], world), "unit": "GB/s",
                    "h2d_bytes_per_step": rd["h2d_bytes"], "d2h_bytes_per_step": rd["d2h_bytes"]},
            "gpu_launches": rd["launches"]}
    if not args.no_extensions and not is_decode(w) and w.name == gi.GQA_PREFILL.name:
        # the extension rows: sliding-window prefill and short decode chunks
        ws_ = gi.WORKLOADS["swa_prefill"]
        rs = measure_prefill(ws_, max(10, args.steps // 4), max(3, args.warmup), world, dev, 2)
        mss = rs["ms_total"] / max(10, args.steps // 4)
        ach = algorithmic_flops(ws_) / (mss * 1e-3) / 1e12
        line["swa_prefill"] = {
            "metric": "TFLOP/s (window-visible pairs)", "value": throughput(ws_, mss, world),
            "unit": "TFLOP/s", "ms_per_step": mss, "config": workload_config(ws_),
            "roofline": tensor_roofline(ach, peaks, peak_src, clocks, load_traffic("gqa_fwd_sm100_kernel", ws_.name),
                                        "gqa_fwd_sm100_kernel<window>"),
            "gpu_launches": rs["launches"]}
        wc = gi.WORKLOADS["chunk_decode"]
        nst = max(3, args.steps // 20)
        rc_ = measure_decode(wc, nst, max(3, args.warmup), world, dev, 2)
        msc = rc_["ms_total"] / nst
        achc = (kv_bytes(wc) + qo_bytes(wc)) / (msc * 1e-3) / 1e9
        line["chunk_decode"] = {
            "metric": "KV GB/s", "value": throughput(wc, msc, world), "unit": "GB/s", "ms_per_step": msc,
            "config": workload_config(wc, {"splits": rc_["splits"]}),
            "roofline": {"bound": "hbm", "achieved": achc, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achc / peaks["hbm_gbs"], "traffic": load_traffic("gqa_decode_sm100_kernel", wc.name),
                         "peak_source": f"{peak_src} hbm_gbs (copy, read+write bytes)"},
            "gpu_launches": rc_["launches"]}
        # variable-length rows: packed prefill, chunked prefill after cached prefixes,
        # paged decode with per-sequence lengths
        nsv = max(10, args.steps // 4)
        for key in ("varlen_prefill", "chunked_prefill"):
            wv = gi.VARLEN_WORKLOADS[key]
            rv = measure_varlen(wv, nsv, max(3, args.warmup), world, dev)
            msv = rv["ms_total"] / nsv
            achv = varlen_flops(wv) / (msv * 1e-3) / 1e12
            line[key] = {
                "metric": "TFLOP/s (causal-visible pairs of every sequence)", "value": world * achv,
                "unit": "TFLOP/s", "ms_per_step": msv,
                "config": varlen_config(wv) | {"tokens_q": rv["tokens_q"], "tokens_k": rv["tokens_k"]},
                "roofline": tensor_roofline(achv, peaks, peak_src, clocks,
                                            load_traffic("gqa_fwd_sm100_kernel_varlen", wv.name),
                                            "gqa_varlen_plan_kernel + gqa_fwd_sm100_kernel<varlen>"),
                "gpu_launches": rv["launches"]}
        # the chunked-prefill workload again, its keys read from a paged pool
        wv = gi.VARLEN_WORKLOADS["chunked_prefill"]
        rpp = measure_paged_prefill(wv, 64, nsv, max(3, args.warmup), world, dev)
        mspp = rpp["ms_total"] / nsv
        achpp = varlen_flops(wv) / (mspp * 1e-3) / 1e12
        line["paged_chunked_prefill"] = {
            "metric": "TFLOP/s (causal-visible pairs of every sequence)", "value": world * achpp, "unit": "TFLOP/s",
            "ms_per_step": mspp, "config": varlen_config(wv) | {"keys": "paged, 64 per page, seeded random page order"},
            "roofline": tensor_roofline(achpp, peaks, peak_src, clocks, None,
                                        "gqa_varlen_plan_kernel + gqa_fwd_sm100_kernel<varlen, paged>"),
            "gpu_launches": rpp["launches"]}
        # backward (training) on the headline workload
        nsb = max(10, args.steps // 4)
        rb = measure_bwd(w, nsb, max(3, args.warmup), world, dev)
        msb = rb["ms_total"] / nsb
        achb = bwd_flops(w) / (msb * 1e-3) / 1e12
        line["backward"] = {
            "metric": "TFLOP/s (10 * D * Hq * B * causal-visible pairs: S, dP, dV, dK, dQ)", "value": world * achb,
            "unit": "TFLOP/s", "ms_per_step": msb, "config": workload_config(w),
            "roofline": tensor_roofline(achb, peaks, peak_src, clocks,
                                        load_traffic("gqa_bwd_sm100_kernel", w.name),
                                        "gqa_bwd_prep_kernel + gqa_bwd_sm100_kernel + gqa_bwd_dq_kernel"),
            "gpu_launches": rb["launches"]}
        wp = gi.VARLEN_WORKLOADS["paged_decode"]
        nsp = max(3, args.steps // 20)
        rp = measure_paged_decode(wp, nsp, max(3, args.warmup), world, dev)
        msp = rp["ms_total"] / nsp
        achp = paged_kv_bytes(wp) / (msp * 1e-3) / 1e9
        line["paged_decode"] = {
            "metric": "KV GB/s (every cached key of every sequence)", "value": world * achp, "unit": "GB/s",
            "ms_per_step": msp,
            "config": {"workload": wp.name, "B": wp.B, "Hq": wp.Hq, "Hkv": wp.Hkv, "D": wp.D, "Tq": wp.Tq,
                       "cache_len": f"U[{wp.len_lo},{wp.len_hi}]", "page": wp.page,
                       "pool": "[pages, page, Hkv, D], seeded random page order", "splits": rp["splits"]},
            "roofline": {"bound": "hbm", "achieved": achp, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achp / peaks["hbm_gbs"],
                         "traffic": load_traffic("gqa_decode_sm100_kernel_varlen", wp.name),
                         "peak_source": f"{peak_src} hbm_gbs (copy, read+write bytes)"},
            "gpu_launches": rp["launches"]}
    sampler.stop()

    if rank == 0 and world == 1 and not args.no_cpu:
        threads = cpu_threads()
        flops, secs, rows = oracle_sample(w, args.cpu_budget, threads)
        if is_decode(w):
            cv = len(rows) / (w.B * w.Hq * w.Tq) * kv_bytes(w) / secs / 1e9
        else:
            cv = flops / secs / 1e12
        line["cpu_baseline"] = {"value": cv, "unit": unit, "cores": threads, "kind": "oracle",
                                "sample": f"{len(rows)} of {w.B * w.Hq * w.Tq} output rows "
                                          f"(seeded sample, fp64), {secs:.1f} s"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
