"""The multi-GPU form is independent replicas: each rank runs the whole layer
on its own batch, times are maxed over ranks and the throughput counts every
rank's work.  This checks that host logic with two gloo ranks on the CPU."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    local = [10.0 + rank, 5.0 * (rank + 1)]  # per-rank step and GEMM totals (ms)
    got = bench.reduce_max(local)
    tops = bench.job_tops(2 * 2048 * 4096 * 6144, 50, world, got[0])
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, tops))


def test_two_replicas_max_time_and_job_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, tops in res:
        assert got == [11.0, 10.0]  # the slowest rank's times, on every rank
        ops = 2 * 2048 * 4096 * 6144 * 50 * 2
        assert tops == pytest.approx(ops / 11e-3 / 1e12)


def test_single_process_is_identity():
    import bench
    assert bench.reduce_max([3.0, 4.0]) == [3.0, 4.0]
    assert bench.job_tops(10 ** 12, 1, 1, 1000.0) == pytest.approx(1.0)
