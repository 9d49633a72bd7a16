"""Multi-rank host logic of the replica and KV-group-shard paths (gloo, 2 processes on CPU)."""
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


def test_group_plan_covers_every_group_of_every_replica():
    for world, tp in ((1, 1), (2, 2), (4, 4), (4, 2), (8, 4), (8, 2)):
        seen = {}
        for r in range(world):
            rep, g0, ng = replicas.group_plan(r, world, tp)
            seen.setdefault(rep, []).extend(range(g0, g0 + ng))
        assert len(seen) == world // tp
        assert all(v == [0, 1, 2, 3] for v in seen.values())
    for bad in ((0, 2, 3), (0, 3, 2), (2, 2, 2)):
        with pytest.raises(ValueError):
            replicas.group_plan(*bad)


def _heads(nq, g0, ng):
    """A deterministic stand-in output whose every element names its query, head and dim."""
    q = torch.arange(nq, dtype=torch.float32)[:, None, None]
    h = torch.arange(16 * g0, 16 * (g0 + ng), dtype=torch.float32)[None, :, None]
    d = torch.arange(192, dtype=torch.float32)[None, None, :]
    return q * 1e5 + h * 200 + d


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rep, g0, ng = replicas.group_plan(rank, world, tp=world)
        grp = replicas.tp_group(world, world)
        full = replicas.gather_heads(_heads(3, g0, ng), grp, tp=world)
        out[rank] = (g0, ng, bool(torch.equal(full, _heads(3, 0, 4))))
    finally:
        dist.destroy_process_group()


def test_two_group_shards_gather_the_64_heads():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
    assert (out[0][0], out[0][1]) == (0, 2) and (out[1][0], out[1][1]) == (2, 2)
    assert out[0][2] and out[1][2]


def test_assemble_heads_rejects_partial_cover():
    with pytest.raises(ValueError):
        replicas.assemble_heads([_heads(2, 0, 2)])
