"""Multi-process (world size 2, gloo, CPU) check of the replica aggregation that
bench.py uses for N > 1 GPUs: each rank runs its own copy of the workload, the
job time is the slowest rank's, and throughput counts every rank's units. No
data-path collective exists; the only collective is the max of the timings."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    local_ms = [120.0, 150.0][rank]
    slowest = bench.reduce_max(local_ms)
    value = bench.replica_throughput(2048, 10, world, slowest)
    q.put((rank, slowest, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, value in res:
        assert slowest == 150.0
        assert value == pytest.approx(2048 * 10 * 2 / 0.150)


def test_single_process_is_identity():
    import bench

    assert bench.reduce_max(3.5) == 3.5
    assert bench.replica_throughput(2048, 4, 1, 2.0) == pytest.approx(2048 * 4 / 0.002)
