"""Multi-rank host logic of the replica path (gloo, 2 processes on CPU)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_long_context_dsa_b200 import replicas


def test_shard_covers_every_unit_once():
    for n in (0, 1, 7, 32, 33, 1000):
        for world in (1, 2, 3, 8):
            got = [u for r in range(world) for u in replicas.shard(n, r, world)]
            assert got == list(range(n))
            sizes = [len(replicas.shard(n, r, world)) for r in range(world)]
            assert max(sizes) - min(sizes) <= 1


def test_shard_rejects_bad_rank():
    with pytest.raises(ValueError):
        replicas.shard(10, 2, 2)


def test_job_throughput_counts_every_rank():
    assert replicas.job_throughput(1000, 4, 500.0) == 8000.0
    with pytest.raises(ValueError):
        replicas.job_throughput(1, 1, 0.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, _ = replicas.dist_env()
        assert (r, w) == (rank, world)
        replicas.barrier()
        slowest = replicas.max_over_ranks(10.0 + 5.0 * rank)       # rank 1 is the slow one
        units = len(replicas.shard(33, rank, world))
        out[rank] = (slowest, units, replicas.job_throughput(17, world, slowest))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] + out[1][1] == 33
    assert out[0][2] == out[1][2] == 2 * 17 / 0.015
