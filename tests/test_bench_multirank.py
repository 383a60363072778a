"""The bench's multi-rank aggregation on CPU: two gloo ranks, max over ranks, whole-job rate.

On the GPU machine every rank runs its own replica of the step (the path shards into
independent problems, no data-path collective); the only cross-rank steps are the barriers
and the max of the device-timed totals, exercised here with the gloo backend.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [12.5, 20.0][rank]          # per-rank device-timed totals
        dist.barrier()
        slowest = bench.max_over_ranks(my_ms, world, device="cpu")
        rate = bench.aggregate_rate(1e12, world, slowest)
        q.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, rate in got:
        assert slowest == 20.0                       # max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 1e12 / 0.020)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_rate(2.0, 1, 1000.0) == pytest.approx(2.0)
