"""bench.py's JSON line on the CPU: the measurement functions (the only parts that need a GPU)
are replaced by fakes that return fixed timings, and each entry point's line is checked for
the keys and the arithmetic the bench contract asks for. This catches mistakes in the line
assembly that would otherwise only show on a GPU run."""
import json

import pytest

import bench
import gqa_inputs as gi

MS = 2.0  # fake milliseconds per step


def fake_result(steps, e2e_steps=0, long_s=0.0):
    r = {"ms_total": MS * steps, "t0": 0.0, "t1": 1.0, "launches": steps, "splits": 3, "tokens_q": 100,
         "tokens_k": 200, "e2e_ms_total": 10.0 * max(e2e_steps, 1), "e2e_steps": max(e2e_steps, 1),
         "h2d_bytes": 123, "d2h_bytes": 45, "steps": steps}
    if long_s > 0:
        n = int(long_s * 1e3 / MS)
        r.update(long_steps=n, long_ms_total=MS * n, long_t0=0.0, long_t1=1.0)
    return r


# one fake per measurement function, with that function's signature
FAKES = {
    "measure_prefill": lambda w, steps, warmup, world, dev, e2e_steps=0, inputs=None, long_s=0.0:
        fake_result(steps, e2e_steps, long_s),
    "measure_decode": lambda w, steps, warmup, world, dev, e2e_steps=0, inputs=None, long_s=0.0:
        fake_result(steps, e2e_steps, long_s),
    "measure_varlen": lambda w, steps, warmup, world, dev, e2e_steps=0: fake_result(steps, e2e_steps),
    "measure_paged_decode": lambda w, steps, warmup, world, dev, e2e_steps=0: fake_result(steps, e2e_steps),
    "measure_bwd": lambda w, steps, warmup, world, dev: fake_result(steps),
    "measure_paged_prefill": lambda w, page, steps, warmup, world, dev: fake_result(steps),
}


# the oracle's figure for a config row, with the longest sample string it can print
FAKE_CPU = {"value": 0.05434, "unit": "TFLOP/s", "cores": 128, "kind": "oracle",
            "sample": "41234 of 1048576 output rows (seeded sample, fp64), 5.0 s; "
                      "full run extrapolated by visible pairs: 16211 s"}


@pytest.fixture
def fake_gpu(monkeypatch):
    import torch
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    for name, fake in FAKES.items():
        monkeypatch.setattr(bench, name, fake)
    # the config rows make their host inputs (8.6 GB for GQA decode) and run the oracle on them
    monkeypatch.setattr(bench, "make_inputs", lambda w: (None, None, None))
    monkeypatch.setattr(bench, "oracle_baseline", lambda w, budget, threads, inputs=None: dict(FAKE_CPU))


def run_main(capsys, argv):
    bench.main(argv)
    out = capsys.readouterr().out
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out
    return json.loads(lines[-1])


BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
             "vs_baseline", "dtype", "data", "config", "roofline", "gpu_launches", "clocks"}
ROOF_KEYS = {"bound", "achieved", "peak", "unit", "frac", "traffic"}


ROW_ROOF_KEYS = {"achieved", "peak", "frac", "traffic"}  # a row's unit is its value's


def check_roofline(r, rel=1e-12, keys=ROOF_KEYS):
    assert keys <= set(r), r
    assert r["peak"] > 0 and abs(r["frac"] - r["achieved"] / r["peak"]) <= rel * r["frac"]


EXTENSION_ROWS = ("swa_prefill", "chunk_decode", "varlen_prefill", "chunked_prefill", "paged_chunked_prefill",
                  "paged_decode", "backward")
CONFIG_ROWS = ("mqa_long", "mha_suffix", "decode")


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
    assert d["long_pass"]["steps"] * MS >= 1000.0 and d["long_pass"]["clocks"]["scope"]
    # every row, the benchmark configs last (the end of the line is what a log tail keeps)
    assert tuple(d["rows"]) == EXTENSION_ROWS + CONFIG_ROWS
    for key, row in d["rows"].items():
        check_roofline(row["roofline"], rel=1e-3, keys=ROW_ROOF_KEYS)
        assert row["value"] > 0 and abs(row["ms_per_step"] - MS) < 1e-9, key
    for key in CONFIG_ROWS:
        row = d["rows"][key]
        assert "cpu_baseline" not in row and row["workload"]  # --no-cpu
        w = bench.gi.WORKLOADS[dict((k, n) for k, n, _ in bench.CONFIG_ROWS)[key]]
        want = (bench.kv_bytes(w) + bench.qo_bytes(w)) / (MS * 1e-3) / 1e9 if key == "decode" else \
            bench.algorithmic_flops(w) / (MS * 1e-3) / 1e12
        assert abs(row["value"] - want) <= 1e-3 * want, key


def test_default_line_fits_a_log_tail(fake_gpu, capsys):
    """A log keeps the last ~3 KB of the line: all rows must fit there, the three benchmark
    configs within the last 1.4 KB."""
    d = run_main(capsys, ["--steps", "20", "--warmup", "5"])
    for key in CONFIG_ROWS:
        assert d["rows"][key]["cpu_baseline"] == FAKE_CPU
    rows = json.dumps({"rows": d["rows"]})
    assert len(rows) < 2900, len(rows)
    configs = json.dumps({k: d["rows"][k] for k in CONFIG_ROWS})
    assert len(configs) < 1400, len(configs)
    assert json.dumps(d).endswith(json.dumps(d["rows"]) + "}")


def test_default_line_with_the_cpu_baseline(fake_gpu, capsys):
    monkey_out = run_main(capsys, ["--steps", "4", "--warmup", "3", "--no-extensions", "--no-configs",
                                   "--cpu-budget", "0.3"])
    c = monkey_out["cpu_baseline"]
    assert c == FAKE_CPU or (c["kind"] == "oracle" and c["value"] > 0 and c["cores"] >= 1)
    assert "rows" not in monkey_out


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


def test_both_arms_print_the_same_config(fake_gpu, capsys, monkeypatch):
    ours = run_main(capsys, ["--steps", "4", "--warmup", "3", "--no-extensions", "--no-configs", "--no-cpu"])
    monkeypatch.setattr(bench, "oracle_sample", lambda w, budget, threads, q=None, k=None, v=None:
                        (1e9, 1.0, list(range(10))))
    ref = run_main(capsys, ["--impl", "reference", "--steps", "2", "--warmup", "3"])
    assert ref["config"] == ours["config"] and ref["impl"] == "reference"


def test_fakes_keep_the_real_signatures():
    import inspect
    for name, fake in FAKES.items():
        assert list(inspect.signature(getattr(bench, name)).parameters) == list(inspect.signature(fake).parameters)
