"""The bench's multi-rank plumbing on CPU: two gloo ranks, each with its own
independent problem (weak scaling, no data-path collective); the timed value is the
max over ranks and the reported throughput counts every rank's work."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    worst = bench.max_over_ranks(10.0 + rank, w)          # rank 1 is the slower one
    wl = bench.gi.WORKLOADS["gqa_prefill"]
    one = bench.throughput(wl, worst, 1)
    agg = bench.throughput(wl, worst, w)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, worst, one, agg))


def test_two_gloo_ranks_take_the_max_time_and_aggregate_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, one, agg in res:
        assert worst == 11.0
        assert agg == pytest.approx(2 * one)


def _bench_rank(rank, world, port, q):
    """One rank of bench.main with the GPU measurements faked and the process group on gloo."""
    import contextlib
    import io

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from tests.test_bench_line import FAKES
    torch.cuda.set_device = lambda *a, **k: None
    real_init = dist.init_process_group
    dist.init_process_group = lambda backend, timeout=None, device_id=None: real_init("gloo", timeout=timeout)
    for name, fake in FAKES.items():
        setattr(bench, name, fake)
    bench.make_inputs = lambda w: (None, None, None)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main(["--gpus", str(world), "--steps", "4", "--warmup", "3", "--no-extensions"])
    q.put((rank, out.getvalue()))


def test_bench_line_over_two_gloo_ranks():
    import json
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    outs = dict(q.get(timeout=10) for _ in range(2))
    assert outs[1].strip() == ""  # only rank 0 prints
    d = json.loads([l for l in outs[0].splitlines() if l.startswith("{")][-1])
    import bench
    w = bench.gi.WORKLOADS["gqa_prefill"]
    per_rank = bench.algorithmic_flops(w) / (d["ms_per_step"] * 1e-3) / 1e12
    assert d["n_gpus"] == 2 and d["scaling"] == "weak"
    assert d["value"] == pytest.approx(2 * per_rank)
    assert "cpu_baseline" not in d  # the oracle baseline runs at one rank only
    # the benchmark-config rows count both ranks' work too, and carry no oracle figure
    wm = bench.gi.WORKLOADS["mqa_long"]
    row = d["rows"]["mqa_long"]
    assert row["value"] == pytest.approx(2 * bench.algorithmic_flops(wm) / (row["ms_per_step"] * 1e-3) / 1e12,
                                         rel=1e-3)
    assert all("cpu_baseline" not in r for r in d["rows"].values())
