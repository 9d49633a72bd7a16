"""Replica bookkeeping for one process per GPU (weak scaling, no data-path collective).

Decode requests are independent: every rank owns a disjoint set of requests (its own caches,
its own launches), and the ranks meet only to time the job.  The job's time is the slowest
rank's; its throughput counts the units every rank processed.
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def dist_env():
    """(rank, world, local_rank) from the launcher's environment (1 process when unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard(n_units: int, rank: int, world: int) -> range:
    """Units [lo, hi) of `rank` when n_units are split as evenly as possible over `world`
    ranks (contiguous blocks; the first n_units % world ranks get one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return range(lo, lo + base + (1 if rank < extra else 0))


def barrier():
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """The largest x over all ranks (x itself with one process)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, slowest_ms: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    if slowest_ms <= 0:
        raise ValueError("time must be positive")
    return world * units_per_rank / (slowest_ms / 1e3)
