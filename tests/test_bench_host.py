"""bench.py's host-side arithmetic (CPU only): the work counts behind every roofline
figure, checked against brute-force enumeration, and the peak and traffic bookkeeping."""
import json
import os

import numpy as np

import bench
import gqa_inputs as gi


def brute_pairs(Tq, Tk, window=0):
    n = 0
    for i in range(Tq):
        pos = Tk - Tq + i
        lo = max(0, pos - window + 1) if window > 0 else 0
        n += pos - lo + 1
    return n


def test_visible_pairs_match_enumeration():
    for Tq, Tk, w in [(1, 1, 0), (5, 5, 0), (3, 10, 0), (7, 7, 3), (4, 20, 6), (9, 9, 100), (1, 32768, 0)]:
        assert bench.visible_pairs(Tq, Tk, w) == brute_pairs(Tq, Tk, w), (Tq, Tk, w)


def test_flop_and_byte_counts():
    w = gi.WORKLOADS["gqa_prefill"]
    assert bench.algorithmic_flops(w) == 4.0 * 128 * 32 * 4 * (4096 * 4097 // 2)
    assert abs(bench.bwd_flops(w) / bench.algorithmic_flops(w) - 2.5) < 1e-12
    d = gi.WORKLOADS["gqa_decode"]
    assert bench.kv_bytes(d) == 2 * 64 * 8 * 32768 * 128 * 2
    vw = gi.VARLEN_WORKLOADS["chunked_prefill"]
    lq, lk = vw.lengths()
    want = 4.0 * vw.D * vw.Hq * sum(brute_pairs(int(a), int(b)) for a, b in zip(lq, lk))
    assert bench.varlen_flops(vw) == want
    pw = gi.VARLEN_WORKLOADS["paged_decode"]
    assert bench.paged_kv_bytes(pw) == 2 * int(pw.lengths().sum()) * pw.Hkv * pw.D * 2


def test_tensor_peak_is_the_burst_figure():
    peaks = {"bf16_tflops": 1630.1, "bf16_tflops_sustained": 1374.1}
    assert bench.tensor_peak(peaks, "measured") == (1630.1, "measured bf16_tflops (burst; kernel timed alone)")
    assert bench.tensor_peak({"bf16_tflops": 1590.0}, "fallback")[0] == 1590.0


def test_traffic_figures_follow_their_kernel_sources():
    path = os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")
    table = json.load(open(path))
    for kernel, entries in table.items():
        if kernel.startswith("_"):
            continue
        assert kernel in bench.KERNEL_SOURCES
        for workload, e in entries.items():
            got = bench.load_traffic(kernel, workload)
            fresh = e["kernel_source_hash"] == bench.kernel_source_hash(kernel)
            assert (got == e["dram_bytes_per_launch"]) if fresh else got is None
            assert e["dram_bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"]
    assert bench.load_traffic("gqa_fwd_sm100_kernel", "no such workload") is None


def test_tensor_roofline_fractions():
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    r = bench.tensor_roofline(800.0, peaks, "measured", 123, "k")
    assert r["peak"] == 1600.0 and r["frac"] == 0.5 and r["frac_of_sustained"] == 800.0 / 1400.0
    assert r["traffic"] == 123 and r["kernel"] == "k" and r["bound"] == "tensor"


def test_rows_round_to_four_digits():
    r = bench.row_entry(1234.5678, 0.123456, 1234.5678, 1630.1, None, "w", {"value": 1})
    assert r == {"workload": "w", "value": 1235.0, "ms_per_step": 0.1235,
                 "roofline": {"achieved": 1235.0, "peak": 1630.1, "frac": 0.7574, "traffic": None},
                 "cpu_baseline": {"value": 1}}
    assert bench.sig(None) is None and bench.sig(0.000123456) == 0.0001235


def test_oracle_baseline_full_and_extrapolated():
    """All rows when the budget allows; otherwise a sample whose full-run time is
    extrapolated by visible pairs, and labelled so."""
    import dataclasses
    w = gi.TINY
    full = bench.oracle_baseline(w, 30.0, 2)
    assert full["sample"].startswith(f"all {w.B * w.Hq * w.Tq} output rows") and full["value"] > 0
    big = dataclasses.replace(w, Tq=4096, Tk=4096, name="tiny shape, long rows")
    part = bench.oracle_baseline(big, 0.05, 2)
    assert "extrapolated by visible pairs" in part["sample"] and part["unit"] == "TFLOP/s"
    dec = dataclasses.replace(w, Tq=1, Tk=2048, name="tiny decode")
    assert bench.oracle_baseline(dec, 10.0, 2)["unit"] == "GB/s"


def _undefined_globals(path):
    """Names that a function of the module reads as globals but that neither the module
    nor the builtins define (what a static checker reports as an undefined name)."""
    import builtins
    import symtable
    src = open(path, encoding="utf-8").read()
    top = symtable.symtable(src, path, "exec")
    defined = {s.get_name() for s in top.get_symbols() if s.is_assigned() or s.is_imported()}
    defined |= set(dir(builtins)) | {"__file__", "__name__"}
    missing = []

    def walk(tab):
        for sym in tab.get_symbols():
            if sym.is_referenced() and sym.is_global() and sym.get_name() not in defined:
                missing.append((tab.get_name(), tab.get_lineno(), sym.get_name()))
        for child in tab.get_children():
            walk(child)
    for child in top.get_children():
        walk(child)
    return missing


def test_host_scripts_have_no_undefined_names():
    import __graft_entry__
    import grouped_query_softmax_b200 as pkg
    for path in (bench.__file__, __graft_entry__.__file__, pkg.__file__):
        assert _undefined_globals(path) == [], path
