"""The N > 1 path of bench.py on the CPU: two gloo ranks stand for two GPU replicas.

The layer does not shard, so N GPUs run N independent replicas; the job's time is the slowest
rank's (max over ranks) and its throughput counts every rank's tokens.
"""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        slowest = bench.allreduce_max(1.0 + rank, world)   # rank 1 is the slow one
        bench.barrier(world)
        q.put((rank, slowest, bench.job_throughput(256, world, slowest)))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [2.0, 2.0]                 # both ranks agree on the max
    assert res[0][2] == pytest.approx(2 * 256 / 2e-3)         # 512 tokens in 2 ms


def test_single_replica_is_identity():
    assert bench.allreduce_max(3.5, 1) == 3.5
    assert bench.job_throughput(256, 1, 4.0) == pytest.approx(64000.0)
