"""Multi-GPU bookkeeping for one process per GPU.

Two ways to split a decode job:
  * replicas: decode requests are independent, every rank owns a disjoint set of requests
    (its own caches, its own launches) and the ranks meet only to time the job (weak
    scaling, no data-path collective);
  * KV-group shards ([P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: the indexer's regions and
    heads map one to one onto the 4 KV groups): a rank holds the summaries and K/V of
    `4 / tp` groups of every request, runs the `_groups` calls on them, and the 16 heads of
    output per group are gathered across the tp ranks of its replica (one all-gather of the
    step's output); world > 4 ranks form world / 4 replicas of 4 shards.
The job's time is the slowest rank's; its throughput counts the units every replica processed.
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


def group_plan(rank: int, world: int, tp: int) -> tuple:
    """KV-group shard of `rank` when `world` ranks form world / tp replicas of tp shards
    (tp = 1, 2 or 4 ranks per replica, world a multiple of tp).  Returns (replica, g0, ng):
    the rank holds groups g0 .. g0 + ng - 1 (ng = 4 / tp) of the replica's requests; the
    ranks of one replica are consecutive, in group order."""
    if tp not in (1, 2, 4) or world < 1 or world % tp or not 0 <= rank < world:
        raise ValueError("tp must be 1, 2 or 4 and divide world; rank out of range")
    ng = 4 // tp
    return rank // tp, (rank % tp) * ng, ng


def assemble_heads(parts):
    """The [nq][64][192] output of a query batch from its tp shards' [nq][16*ng][192]
    outputs, in group order (shard i holds query heads 16*g0_i .. 16*(g0_i + ng) - 1)."""
    out = torch.cat(list(parts), dim=1)
    if out.shape[1] != 64:
        raise ValueError("the shards must cover the 64 query heads")
    return out


def tp_group(world: int, tp: int):
    """The process group of this rank's replica (ranks r // tp * tp .. + tp - 1); every rank
    creates every replica's group, in the same order, as torch.distributed requires."""
    mine = None
    rank = dist.get_rank()
    for r0 in range(0, world, tp):
        g = dist.new_group(list(range(r0, r0 + tp)))
        if r0 <= rank < r0 + tp:
            mine = g
    return mine


def gather_heads(local: torch.Tensor, group=None, tp: int = 1) -> torch.Tensor:
    """All-gather of the shards' outputs [nq][16*ng][192] over the replica's process group
    (NCCL on GPUs, gloo on CPU): every rank of the replica gets the full [nq][64][192]."""
    if tp == 1:
        return local
    parts = [torch.empty_like(local) for _ in range(tp)]
    dist.all_gather(parts, local.contiguous(), group=group)
    return assemble_heads(parts)
