"""Host logic of the multi-GPU benchmark path on CPU: two gloo ranks (the
same calls bench.py makes over NCCL), each with its own timing; the job's time
is the slowest rank's and the job's throughput counts every rank's replica."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, lr = bench.rank_env()
    assert (r, w, lr) == (rank, world, rank)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(my_ms, torch.device("cpu"))
        value = bench.job_throughput(16.06e9, world, 20, got)
        dist.barrier()
        out.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, value in res:
        assert got == 15.0  # both ranks see the slowest rank's time
        assert value == pytest.approx(2 * 16.06e9 * 20 / 0.015 / 1e9)


def test_single_rank_is_identity():
    import torch
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_throughput(1e9, 1, 10, 1000.0) == pytest.approx(10.0)
