#!/usr/bin/env python
"""Benchmark of causal grouped-query softmax attention on B200.

One step = one pass of the hot path over one batch of synthetic input. The main line is
gqa_attn_fwd on the GQA prefill workload (B4 Hq32 Hkv8 T4096 D128), metric TFLOP/s with
FLOPs = 4 * D * Hq * B * (causal-visible query/key pairs), timed over exactly --steps
steps with inputs resident in HBM; a second pass of at least --long-pass seconds gives the
clock record a long window; "e2e" is the host-memory call gqa_attn_fwd_host end to end.

"rows" holds the other measurements, each its own step timed alone, the benchmark configs
last: the extension workloads (sliding window, verify chunk, variable-length, paged,
backward), then MQA long prefill (B1 Hq32 Hkv1 T32768), MHA suffix (B8 H16 Tq512 over
Tk8192, Q x 4) and GQA decode (B64 Hq32 Hkv8 Tk32768; KV GB/s = (K + V bytes) / time),
each of these three with the fp64 oracle's time on the host cores beside it.

Inputs are seeded iid N(0,1) rounded to bf16 (see gqa_inputs). Under torchrun every rank
runs its own copy of the workload (independent problems, no data-path collective): weak
scaling, value = all ranks' work / max-over-ranks time.

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

L2_NOTE = "inputs larger than L2 (no flush)"
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


def tensor_peak(peaks, peak_src):
    """(peak, description): every kernel here is timed alone, so the burst GEMM figure."""
    return peaks["bf16_tflops"], f"{peak_src} bf16_tflops (burst; kernel timed alone)"


def tensor_roofline(achieved, peaks, peak_src, traffic, kernel):
    """The roofline object of a tensor-bound main line: the fraction of the burst peak,
    with the fractions of the sustained (power-capped) and 2250 TFLOP/s spec figures for
    context."""
    peak, src = tensor_peak(peaks, peak_src)
    sustained = peaks.get("bf16_tflops_sustained", peak)
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic, "peak_source": src,
            "frac_of_sustained": achieved / sustained, "frac_of_spec_2250": achieved / 2250.0, "kernel": kernel}


def sig(x, n: int = 4):
    """x to n significant digits (keeps the JSON line short); None stays None."""
    return None if x is None else float(f"{x:.{n}g}")


def row_entry(value, ms, achieved, peak, traffic, workload=None, cpu=None):
    """One sub-row of the bench line: throughput, time per step and the roofline of its
    dominant kernel (achieved / peak in the row's own unit; traffic = DRAM bytes per launch
    from a committed ncu capture, or None)."""
    r = {} if workload is None else {"workload": workload}
    r.update({"value": sig(value), "ms_per_step": sig(ms),
              "roofline": {"achieved": sig(achieved), "peak": peak, "frac": sig(achieved / peak),
                           "traffic": traffic}})
    if cpu is not None:
        r["cpu_baseline"] = cpu
    return r


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
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled while it works.

    NVML is polled every millisecond from a thread (its calls release the GIL), so even
    a 10 ms timed region holds several samples; without NVML, nvidia-smi is sampled every
    50 ms instead. Samples are (wall time, sm MHz, max sm MHz, set of active reasons)."""

    def __init__(self, gpu_id: str | None, dev_index: int | None = None, interval_s: float = 0.001):
        self.samples = []
        self.proc = None
        self.gpu_id = gpu_id
        self.dev_index = dev_index
        self.interval_s = interval_s
        self.source = "none"
        self._stop = threading.Event()

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:  # the CUDA device's own UUID is immune to CUDA_VISIBLE_DEVICES remapping
            import torch
            uuid = str(torch.cuda.get_device_properties(self.dev_index or 0).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu_id or 0))

    def start(self):
        try:
            nv, h = self._nvml_handle()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            return self._start_smi()
        self.source = f"nvml every {self.interval_s * 1e3:g} ms"

        def poll():
            while not self._stop.is_set():
                try:
                    sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    word = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    break
                self.samples.append((time.time(), sm, smax, {n for n, b in bits.items() if word & b}))
                time.sleep(self.interval_s)
        threading.Thread(target=poll, daemon=True).start()

    def _start_smi(self):
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        cmd = ["nvidia-smi", f"--query-gpu={fields}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.gpu_id is not None:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi every 50 ms"

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        def read():
            for line in self.proc.stdout:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 6:
                    active = {REASON_NAMES[i] for i in range(4) if parts[2 + i].lower().startswith("active")}
                    self.samples.append((time.time(), num(parts[0]), num(parts[1]), active))
        threading.Thread(target=read, daemon=True).start()

    def stop(self):
        self._stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        """Median SM clock and every reason seen between t0 and t1 (wall time)."""
        window = [s for s in self.samples if t0 <= s[0] <= t1]
        scope = "timed region"
        if len(window) < 3:
            window = list(self.samples)
            scope = "whole run (timed region shorter than the sampling interval)"
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "scope": "unavailable"}
        sm = [s[1] for s in window if s[1] is not None]
        smax = [s[2] for s in window if s[2] is not None]
        reasons = sorted(set().union(*(s[3] for s in window)))
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(window), "scope": scope, "source": self.source}


def make_sampler(local: int, world: int) -> ClockSampler:
    """A started sampler for this rank's GPU (CUDA device `local`)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_id = vis.split(",")[local] if vis else str(local)
    s = ClockSampler(gpu_id, local)
    s.start()
    time.sleep(0.2)
    return s


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


def long_pass(fn, res, long_s, world, dev):
    """A second timed pass of the same step lasting at least long_s seconds, so the clock
    sampler sees it; its step count follows from the first pass (the same on every rank)."""
    if long_s <= 0:
        return
    ms_step = res["ms_total"] / res["steps"]
    n = max(res["steps"], int(math.ceil(long_s * 1e3 / max(ms_step, 1e-6))))
    ms, t0, t1 = timed(fn, n, 0, world, dev)
    res.update(long_steps=n, long_ms_total=ms, long_t0=t0, long_t1=t1)


def measure_prefill(w, steps, warmup, world, dev, e2e_steps=0, inputs=None, long_s=0.0):
    """attn_fwd (gqa_attn_fwd_split, which splits the last wave's key tiles over the SMs when
    its plan says so, and is gqa_attn_fwd otherwise) over `steps` calls on inputs resident in
    HBM, its workspace allocated once; optionally a long pass of the same call, and the
    host-memory call end to end (e2e_steps > 0)."""
    import torch
    import grouped_query_softmax_b200 as gqa
    q, k, v = inputs if inputs is not None else w.make()
    qd, kd, vd = to_device(q, dev), to_device(k, dev), to_device(v, dev)
    od = torch.empty_like(qd)
    need = gqa.gqa_attn_fwd_split_workspace_bytes(w.B, w.Hq, w.Hkv, w.Tq, w.Tk, w.D, w.window)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    fn = lambda: gqa.attn_fwd(qd, kd, vd, out=od, window=w.window, workspace=ws)
    ms, t0, t1 = timed(fn, steps, warmup, world, dev)
    # a split launch is the forward kernel and the merge of the pieces
    res = {"ms_total": ms, "t0": t0, "t1": t1, "launches": steps * (2 if need else 1), "steps": steps,
           "split_bytes": need}
    long_pass(fn, res, long_s, world, dev)
    st = gqa.gqa_get_device_error(torch.cuda.current_stream().cuda_stream)
    if st != gqa.GQA_OK:
        raise RuntimeError(f"device error after prefill timing: {gqa.gqa_status_string(st)}")
    del qd, kd, vd, od, ws
    torch.cuda.empty_cache()
    if e2e_steps <= 0:
        return res

    # end to end through the public host-memory call (gqa_attn_fwd_host): pinned host inputs
    # in, host output out, every step; its device workspace is allocated once, outside
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


def measure_decode(w, steps, warmup, world, dev, e2e_steps=0, inputs=None, long_s=0.0):
    """gqa_attn_decode(_ex) over `steps` calls on a cache resident in HBM; optionally a long
    pass, and end to end with the inputs copied from pinned host memory every step."""
    import torch
    import grouped_query_softmax_b200 as gqa
    q, k, v = inputs if inputs is not None else w.make()
    qd, kd, vd = to_device(q, dev), to_device(k, dev), to_device(v, dev)
    od = torch.empty_like(qd)
    splits = gqa.gqa_attn_decode_ex_num_splits(w.B, w.Hq, w.Hkv, w.Tq, w.Tk, w.D, w.window, 0)
    need = gqa.gqa_attn_decode_ex_workspace_bytes(w.B, w.Hq, w.Hkv, w.Tq, w.Tk, w.D, w.window, 0)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    fn = lambda: gqa.attn_decode(qd, kd, vd, out=od, workspace=ws, window=w.window)
    ms, t0, t1 = timed(fn, steps, warmup, world, dev)
    res = {"ms_total": ms, "t0": t0, "t1": t1, "splits": splits, "steps": steps,
           "launches": steps * (1 if splits == 1 else 2)}
    long_pass(fn, res, long_s, world, dev)
    st = gqa.gqa_get_device_error(torch.cuda.current_stream().cuda_stream)
    if st != gqa.GQA_OK:
        raise RuntimeError(f"device error after decode timing: {gqa.gqa_status_string(st)}")
    if e2e_steps > 0:
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


def oracle_baseline(w, budget_s: float, threads: int, inputs=None):
    """The fp64 oracle on the host cores, on workload w: every output row when that takes
    about budget_s seconds or less, else a seeded row sample whose time is extrapolated to
    the whole workload by visible pairs (and labelled so). A reported baseline."""
    q, k, v = inputs if inputs is not None else w.make()
    flops, secs, rows = oracle_sample(w, budget_s, threads, q, k, v)
    total = w.B * w.Hq * w.Tq
    if is_decode(w):
        value, unit = len(rows) / total * kv_bytes(w) / secs / 1e9, "GB/s"
    else:
        value, unit = flops / secs / 1e12, "TFLOP/s"
    if len(rows) >= total:
        sample = f"all {total} output rows (fp64), {secs:.1f} s"
    else:
        sample = (f"{len(rows)} of {total} output rows (seeded sample, fp64), {secs:.1f} s; "
                  f"full run extrapolated by visible pairs: {secs * algorithmic_flops(w) / flops:.0f} s")
    return {"value": sig(value), "unit": unit, "cores": threads, "kind": "oracle", "sample": sample}


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
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the rows of the other benchmark configs (MQA long, MHA suffix, GQA decode)")
    ap.add_argument("--no-extensions", action="store_true",
                    help="skip the sliding-window, decode-chunk and variable-length measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--backward", action="store_true",
                    help="measure only the backward pass of the main (dense) workload, e.g. for profiling")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work on the main workload")
    ap.add_argument("--long-pass", type=float, default=1.0,
                    help="seconds of a second timed pass of the main step, long enough for the clock record")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the main workload's batch size / sequence count (for profiling a smaller case)")
    return ap.parse_args(argv)


def workload_config(w, extra=None):
    """The config object of a dense workload; both bench arms print the same one."""
    c = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Tq": w.Tq, "Tk": w.Tk, "D": w.D,
         "q_scale": 2 ** w.q_pow2, "seed": w.seed, "causal": True, "l2": L2_NOTE}
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
    sampler = make_sampler(local, world)
    r = measure_bwd(w, args.steps, args.warmup, world, dev)
    ms_step = r["ms_total"] / args.steps
    achieved = bwd_flops(w) / (ms_step * 1e-3) / 1e12
    clocks = sampler.summary(r["t0"], r["t1"])
    sampler.stop()
    line = {"metric": "GQA attn backward TFLOP/s on 1 B200, % of roofline", "value": world * achieved,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, {"pass": "backward (dQ, dK, dV)"}),
            "roofline": tensor_roofline(achieved, peaks, peak_src, load_traffic("gqa_bwd_sm100_kernel", w.name),
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
    sampler = make_sampler(local, world)
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
        roof = tensor_roofline(achieved, peaks, peak_src, load_traffic("gqa_fwd_sm100_kernel_varlen", w.name),
                               kernel)
    else:
        roof = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": load_traffic("gqa_decode_sm100_kernel_varlen", w.name), "peak_source": src,
                "kernel": kernel}
    line = {"metric": metric, "value": world * achieved, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config | {"l2": L2_NOTE},
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


# The other benchmark configs, measured as rows of the default line (last in it), each with
# the oracle's time on the host cores beside it: (key, workload, oracle seconds).
CONFIG_ROWS = (("mqa_long", "mqa_long", 5.0), ("mha_suffix", "mha_suffix", 12.0), ("decode", "gqa_decode", 3.0))


def hbm_row(work_bytes, ms, peaks, traffic, workload=None, cpu=None, world=1):
    gbs = work_bytes / (ms * 1e-3) / 1e9
    return row_entry(world * gbs, ms, gbs, peaks["hbm_gbs"], traffic, workload, cpu)


def tensor_row(flops, ms, peaks, traffic, workload=None, cpu=None, world=1):
    tf = flops / (ms * 1e-3) / 1e12
    return row_entry(world * tf, ms, tf, peaks["bf16_tflops"], traffic, workload, cpu)


def extension_rows(args, w, world, dev, peaks):
    """The rows of the extension workloads: sliding window, verify chunk, variable-length,
    paged and backward (each its own step, timed alone)."""
    rows = {}
    warm = max(3, args.warmup)
    nsv = max(10, args.steps // 4)   # prefill-sized rows
    nsd = max(3, args.steps // 20)   # decode-sized rows (8 GB of cache per step)
    ws_ = gi.WORKLOADS["swa_prefill"]
    r = measure_prefill(ws_, nsv, warm, world, dev)
    rows["swa_prefill"] = tensor_row(algorithmic_flops(ws_), r["ms_total"] / nsv, peaks,
                                     load_traffic("gqa_fwd_sm100_kernel", ws_.name), world=world)
    wc = gi.WORKLOADS["chunk_decode"]
    r = measure_decode(wc, nsd, warm, world, dev)
    rows["chunk_decode"] = hbm_row(kv_bytes(wc) + qo_bytes(wc), r["ms_total"] / nsd, peaks,
                                   load_traffic("gqa_decode_sm100_kernel", wc.name), world=world)
    for key in ("varlen_prefill", "chunked_prefill"):
        wv = gi.VARLEN_WORKLOADS[key]
        r = measure_varlen(wv, nsv, warm, world, dev)
        rows[key] = tensor_row(varlen_flops(wv), r["ms_total"] / nsv, peaks,
                               load_traffic("gqa_fwd_sm100_kernel_varlen", wv.name), world=world)
    # the chunked-prefill workload again, its keys read from a paged pool of 64-key pages
    wv = gi.VARLEN_WORKLOADS["chunked_prefill"]
    r = measure_paged_prefill(wv, 64, nsv, warm, world, dev)
    rows["paged_chunked_prefill"] = tensor_row(varlen_flops(wv), r["ms_total"] / nsv, peaks, None, world=world)
    wp = gi.VARLEN_WORKLOADS["paged_decode"]
    r = measure_paged_decode(wp, nsd, warm, world, dev)
    rows["paged_decode"] = hbm_row(paged_kv_bytes(wp), r["ms_total"] / nsd, peaks,
                                   load_traffic("gqa_decode_sm100_kernel_varlen", wp.name), world=world)
    # backward (dQ, dK, dV) of the GQA prefill workload
    r = measure_bwd(w, nsv, warm, world, dev)
    rows["backward"] = tensor_row(bwd_flops(w), r["ms_total"] / nsv, peaks,
                                  load_traffic("gqa_bwd_sm100_kernel", w.name), world=world)
    return rows


def make_inputs(w):
    """Host (q, k, v) bf16 bit arrays of a dense workload, shared by the GPU row and the oracle."""
    return w.make()


def config_rows(args, w, world, dev, peaks, with_cpu):
    """The benchmark configs other than the main one (MQA long, MHA suffix, GQA decode),
    each with the oracle beside it on rank 0 at N = 1."""
    rows = {}
    threads = cpu_threads()
    for key, name, budget in CONFIG_ROWS:
        wr = gi.WORKLOADS[name]
        if wr.name == w.name:
            continue
        inputs = make_inputs(wr)
        if is_decode(wr):
            n = max(3, args.steps // 20)
            r = measure_decode(wr, n, max(3, args.warmup), world, dev, inputs=inputs)
        else:
            n = max(10, args.steps // 4)
            r = measure_prefill(wr, n, max(3, args.warmup), world, dev, inputs=inputs)
        cpu = oracle_baseline(wr, budget, threads, inputs) if with_cpu else None
        del inputs
        ms = r["ms_total"] / n
        if is_decode(wr):
            rows[key] = hbm_row(kv_bytes(wr) + qo_bytes(wr), ms, peaks,
                                load_traffic("gqa_decode_sm100_kernel", wr.name), wr.name, cpu, world)
        else:
            rows[key] = tensor_row(algorithmic_flops(wr), ms, peaks,
                                   load_traffic("gqa_fwd_sm100_kernel", wr.name), wr.name, cpu, world)
    return rows


def short_clocks(c):
    return {k: c.get(k) for k in ("sm_mhz", "reasons", "samples", "scope")}


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
    sampler = make_sampler(local, world)

    metric, unit = metric_of(w)
    measure = measure_decode if is_decode(w) else measure_prefill
    r = measure(w, args.steps, args.warmup, world, dev, args.e2e_steps, long_s=args.long_pass)
    ms_step = r["ms_total"] / args.steps
    value = throughput(w, ms_step, world)
    clocks = sampler.summary(r["t0"], r["t1"])

    if is_decode(w):
        achieved = (kv_bytes(w) + qo_bytes(w)) / (ms_step * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": load_traffic("gqa_decode_sm100_kernel", w.name),
                "peak_source": f"{peak_src} hbm_gbs (copy, read+write bytes)",
                "kernel": "gqa_decode_sm100_kernel + gqa_decode_combine_kernel (one call per step)"}
    else:
        achieved = algorithmic_flops(w) / (ms_step * 1e-3) / 1e12
        roof = tensor_roofline(achieved, peaks, peak_src, load_traffic("gqa_fwd_sm100_kernel", w.name),
                               "gqa_fwd_sm100_kernel")

    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w),
            "roofline": roof, "gpu_launches": r["launches"], "clocks": clocks}
    if args.e2e_steps > 0:
        e2e_ms = r["e2e_ms_total"] / r["e2e_steps"]
        line["e2e"] = {"value": throughput(w, e2e_ms, world), "unit": unit, "h2d_bytes_per_step": r["h2d_bytes"],
                       "d2h_bytes_per_step": r["d2h_bytes"], "ms_per_step": e2e_ms, "steps": r["e2e_steps"],
                       "call": ("gqa_attn_decode_ex after host-to-device copies of q, k, v" if is_decode(w) else
                                "gqa_attn_fwd_host: pinned host q, k, v, o; query-row chunks overlap copies "
                                "and kernels")}
    if "long_steps" in r:
        lms = r["long_ms_total"] / r["long_steps"]
        line["long_pass"] = {"steps": r["long_steps"], "ms_per_step": lms, "value": throughput(w, lms, world),
                             "clocks": short_clocks(sampler.summary(r["long_t0"], r["long_t1"]))}

    with_cpu = rank == 0 and world == 1 and not args.no_cpu
    rows = {}
    if not args.no_extensions and w.name == gi.GQA_PREFILL.name:
        rows.update(extension_rows(args, w, world, dev, peaks))
    if not args.no_configs:
        rows.update(config_rows(args, w, world, dev, peaks, with_cpu))
    sampler.stop()

    if with_cpu:
        line["cpu_baseline"] = oracle_baseline(w, args.cpu_budget, cpu_threads())
    if rows:
        line["rows"] = rows
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
