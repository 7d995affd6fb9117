"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): the timed duration is
the maximum over ranks and the reported throughput aggregates every rank's replica stream."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 100.0 + 50.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(ms, world)
        v = bench.aggregate_frames_per_s(world, 10, 320, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_aggregate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v in res:
        assert m == 150.0
        assert v == pytest.approx(2 * 10 * 320 / 0.150)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.aggregate_frames_per_s(1, 4, 320, 1000.0) == pytest.approx(1280.0)
