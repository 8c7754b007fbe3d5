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


def _dying_worker(rank, world, port, q):
    import datetime
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(3)  # leaves between steps: before the reduction of the step timer
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, torch.device("cpu"))
        q.put(("no error", time.time() - t0))
    except Exception as e:  # noqa: BLE001 -- any error type: what matters is that the wait ends
        q.put((type(e).__name__, time.time() - t0))
    q.close()
    q.join_thread()
    os._exit(0)  # no destroy_process_group: its peer is gone


def test_rank_that_leaves_ends_the_others_with_an_error():
    """A rank that exits before the timer's reduction: the remaining rank's
    collective ends with an error within the process group's timeout (5 s
    here) instead of waiting for good."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        what, seconds = q.get(timeout=120)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    assert what != "no error"
    assert seconds < 60
    assert procs[1].exitcode == 3


def test_single_rank_throughput():
    assert bench.aggregate_throughput(1, 2 * 10 ** 12, 1000.0) == pytest.approx(2.0)


def test_bench_reference_arm_under_torchrun():
    """`bench.py --impl reference` launched like the multi-GPU bench (torchrun,
    two ranks, rendezvous on 127.0.0.1): rank 0 alone runs the oracle and
    prints one JSON line with the contract's keys; the other rank exits 0
    without work.  Runs on the CPU (the reference arm needs no GPU)."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(29600 + os.getpid() % 300),
           os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2", "--workload",
           "activation_quantizer", "--steps", "1", "--warmup", "1", "--cpu-seconds", "0.5"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
