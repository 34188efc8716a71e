"""The N-GPU path of bench.py on CPU: world-size-2 `gloo` ranks.

The layer does not shard (replicas only), so the multi-rank logic is the
host side: every rank's timed span is reduced to the maximum, the job's
throughput counts every replica's units, and only rank 0 prints (the
reference arm exits at once on the other ranks).
"""
import datetime
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank "measured" a different time; all must end with the slowest
        got = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
        # a second reduction in the same order (bench reduces the timed and the e2e spans)
        got2 = bench.max_over_ranks(3.0 - rank, "cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()
    results[rank] = (got, got2)


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(results) == {0: (15.0, 3.0), 1: (15.0, 3.0)}


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, "cpu") == 7.5


def test_job_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    # 2 replicas x 2048 tokens x 10 steps in 15 ms
    assert bench.job_throughput(2, 2048, 10, 15.0) == pytest.approx(2 * 2048 * 10 / 0.015)


def test_reference_arm_is_rank0_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(type("A", (), {"steps": 1, "warmup": 1})())
    assert buf.getvalue() == ""
