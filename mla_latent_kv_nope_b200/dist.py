"""Host-side multi-GPU logic of the decode step: one process per GPU.

Sequences are independent, so the batch shards across ranks with no
collective on the data path: each rank decodes its own B sequences (its own
seeded inputs) and the job's throughput is the sum over ranks.  The only
collectives are for timing: a barrier on both sides of the timed region and
the maximum over ranks of the elapsed time (the job is as slow as its
slowest rank).  Works with any torch.distributed backend (NCCL on GPUs, gloo
for the CPU tests).
"""
from __future__ import annotations

import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankEnv:
    rank: int
    world: int
    local_rank: int


def rank_env() -> RankEnv:
    """Rank, world size and local rank from the launcher's environment."""
    return RankEnv(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                   int(os.environ.get("LOCAL_RANK", "0")))


def shard(workload, rank: int):
    """This rank's share of the job: the same shapes with its own input
    stream (seed = rank), i.e. B different sequences per rank."""
    return workload.scaled(seed=workload.seed + rank)


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest x over all ranks (every rank gets it)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank decodes its own tokens each step; the
    step time is the slowest rank's."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)
