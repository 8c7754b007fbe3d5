"""World-size-2 checks of the multi-rank host logic of bench.py on CPU (gloo):
every rank runs its own replica, the timer is reduced with MAX, and the
whole-job throughput counts all ranks' work against the slowest rank."""
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
        local_ms = [12.5, 20.0, 7.0, 9.0][rank]
        ms = bench.max_over_ranks(local_ms, torch.device("cpu"))
        value = bench.aggregate_throughput(world, 10 ** 12, ms)
        dist.barrier()
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_max_over_ranks_and_weak_scaling(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    expect_ms = max([12.5, 20.0, 7.0, 9.0][:world])
    for _, ms, value in res:
        assert ms == expect_ms
        assert value == pytest.approx(world * 1.0 / (expect_ms * 1e-3))


def test_single_rank_throughput():
    assert bench.aggregate_throughput(1, 2 * 10 ** 12, 1000.0) == pytest.approx(2.0)
