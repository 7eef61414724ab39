"""Multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

The GDN path shards without any data exchange (every (batch, value head) scan
is independent), so N GPUs run N independent replicas; the only cross-rank
step is the timing reduction: the job's time per step is the slowest rank's,
and the whole-job rate counts the units of every rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        info = bench.rank_info()
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))  # rank 1 is slower
        rate = bench.job_rate(8192, world, ms)
        q.put((rank, info, ms, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, info, ms, rate in out:
        assert info == (rank, rank, world)
        assert ms == 15.0
        assert rate == pytest.approx(2 * 8192 / 0.015)


def test_single_process_defaults(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.rank_info() == (0, 0, 1)
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_rate(100, 1, 10.0) == pytest.approx(10_000.0)
