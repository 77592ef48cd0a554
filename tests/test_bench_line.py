"""bench.py's JSON line on the CPU: the measurement functions (the only parts that need a GPU)
are replaced by fakes that return fixed timings, and each entry point's line is checked for
the keys and the arithmetic the bench contract asks for. This catches mistakes in the line
assembly that would otherwise only show on a GPU run."""
import json

import pytest

import bench
import gqa_inputs as gi

MS = 2.0  # fake milliseconds per step


def fake_result(steps, e2e_steps=0):
    return {"ms_total": MS * steps, "t0": 0.0, "t1": 1.0, "launches": steps, "splits": 3, "tokens_q": 100,
            "tokens_k": 200, "e2e_ms_total": 10.0 * max(e2e_steps, 1), "e2e_steps": max(e2e_steps, 1),
            "h2d_bytes": 123, "d2h_bytes": 45}


# one fake per measurement function, with that function's signature
FAKES = {
    "measure_prefill": lambda w, steps, warmup, world, dev, e2e_steps: fake_result(steps, e2e_steps),
    "measure_decode": lambda w, steps, warmup, world, dev, e2e_steps: fake_result(steps, e2e_steps),
    "measure_varlen": lambda w, steps, warmup, world, dev, e2e_steps=0: fake_result(steps, e2e_steps),
    "measure_paged_decode": lambda w, steps, warmup, world, dev, e2e_steps=0: fake_result(steps, e2e_steps),
    "measure_bwd": lambda w, steps, warmup, world, dev: fake_result(steps),
    "measure_paged_prefill": lambda w, page, steps, warmup, world, dev: fake_result(steps),
}


@pytest.fixture
def fake_gpu(monkeypatch):
    import torch
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    for name, fake in FAKES.items():
        monkeypatch.setattr(bench, name, fake)


def run_main(capsys, argv):
    bench.main(argv)
    out = capsys.readouterr().out
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out
    return json.loads(lines[-1])


BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
             "vs_baseline", "dtype", "data", "config", "roofline", "gpu_launches", "clocks"}
ROOF_KEYS = {"bound", "achieved", "peak", "unit", "frac", "traffic"}


def check_roofline(r):
    assert ROOF_KEYS <= set(r), r
    assert r["peak"] > 0 and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12


def test_default_line(fake_gpu, capsys):
    d = run_main(capsys, ["--steps", "4", "--warmup", "3", "--no-cpu", "--e2e-steps", "2"])
    assert BASE_KEYS <= set(d)
    w = gi.WORKLOADS["gqa_prefill"]
    assert d["ms_per_step"] == MS and d["steps"] == 4 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert abs(d["value"] - bench.algorithmic_flops(w) / (MS * 1e-3) / 1e12) < 1e-6
    check_roofline(d["roofline"])
    assert d["roofline"]["bound"] == "tensor" and d["config"]["workload"] == w.name
    e = d["e2e"]
    assert {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"} <= set(e) and e["unit"] == d["unit"]
    for row in ("decode", "swa_prefill", "chunk_decode", "varlen_prefill", "chunked_prefill",
                "paged_chunked_prefill", "backward", "paged_decode"):
        assert row in d, row
        check_roofline(d[row]["roofline"])
        assert d[row]["gpu_launches"] > 0


def test_default_line_with_the_cpu_baseline(fake_gpu, capsys):
    d = run_main(capsys, ["--steps", "4", "--warmup", "3", "--no-extensions", "--no-decode", "--cpu-budget", "0.3"])
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["value"] > 0 and c["cores"] >= 1 and c["unit"] == d["unit"]


def test_backward_line(fake_gpu, capsys):
    d = run_main(capsys, ["--backward", "--steps", "5", "--warmup", "3"])
    assert BASE_KEYS <= set(d)
    w = gi.WORKLOADS["gqa_prefill"]
    assert abs(d["value"] - bench.bwd_flops(w) / (MS * 1e-3) / 1e12) < 1e-6
    check_roofline(d["roofline"])


@pytest.mark.parametrize("workload", ["varlen_prefill", "chunked_prefill", "paged_decode"])
def test_varlen_lines(fake_gpu, capsys, workload):
    d = run_main(capsys, ["--workload", workload, "--steps", "5", "--warmup", "3", "--e2e-steps", "1"])
    assert BASE_KEYS <= set(d)
    check_roofline(d["roofline"])
    assert d["roofline"]["bound"] == ("hbm" if workload == "paged_decode" else "tensor")
    assert "e2e" in d


def test_fakes_keep_the_real_signatures():
    import inspect
    for name, fake in FAKES.items():
        assert list(inspect.signature(getattr(bench, name)).parameters) == list(inspect.signature(fake).parameters)
