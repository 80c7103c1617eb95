"""Multi-rank plumbing of the benchmark on CPU (gloo, world size 2).

Every (b, h) of the workload is independent, so under torchrun each rank
runs its own replica with no collective on the data path; the only
collectives are the timing reductions.  These tests run them on CPU ranks.
"""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports times (r + 1, 10 - r): the job takes the slowest rank
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank])
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_timing_is_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res[0] == [2.0, 10.0] and res[1] == [2.0, 10.0]


def test_single_rank_reduction_is_identity():
    assert bench.max_over_ranks([3.5, 1.0]) == [3.5, 1.0]


def test_job_throughput_counts_every_rank():
    # 2 ranks x 4096 tokens x 10 steps in 20 ms (slowest rank)
    assert bench.job_throughput(2, 4096, 10, 20.0) == pytest.approx(2 * 4096 * 10 / 0.020)


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    ns = type("A", (), {"steps": 1, "warmup": 0, "workload": 2})()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(ns)
    assert buf.getvalue() == ""


def test_percentiles_nearest_rank():
    import bench
    q = bench.percentiles([5.0, 1.0, 3.0, 2.0, 4.0, 6.0, 7.0, 8.0, 9.0, 10.0, 11.0])
    assert q == {"p10": 2.0, "median": 6.0, "p90": 10.0}
    assert bench.percentiles([2.5]) == {"p10": 2.5, "median": 2.5, "p90": 2.5}
    assert bench.percentiles([]) == {"p10": None, "median": None, "p90": None}
