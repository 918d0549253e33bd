"""The N > 1 host logic of bench.py, on CPU with two gloo ranks.

The layer does not shard (one GPU quantizes one layer), so several GPUs run
independent replicas: there is no collective on the data path, only the
barrier around the timed region and the max over ranks of the device time.
These tests run that logic with world_size 2 over gloo, no GPU involved.
"""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        dist.barrier()
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world)     # rank 1 is the slow one
        v = bench.job_throughput(world, 4096 * 4096, 3, ms)
        dist.barrier()
        q.put((rank, ms, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_the_job_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, v in got:
        assert ms == 15.0
        assert v == pytest.approx(world * 4096 * 4096 * 3 / 0.015)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.job_throughput(1, 100, 10, 1000.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup, workload, tokens = 1, 0, "layer256", 0

    bench.run_reference(A(), rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(capsys):
    """The oracle arm's JSON line: the contract's keys, the host-only e2e leg
    (no copies) and a sample no larger than the workload."""
    sys.path.insert(0, ROOT)
    import json
    import bench

    class A:
        steps, warmup, workload, tokens = 1, 0, "layer256", 0

    bench.run_reference(A(), rank=0, world=1)
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "H on 2048 of 2048 tokens (time x1)" in cb["sample"]
    assert "64 of 256 rows (time x4)" in cb["sample"]
