"""Host-side multi-GPU logic of the decode step: one process per GPU.

Batch sharding (the default): sequences are independent, so the batch shards
across ranks with no collective on the data path: each rank decodes its own
B sequences (its own seeded inputs) and the job's throughput is the sum over
ranks.  The only collectives are for timing: a barrier on both sides of the
timed region and the maximum over ranks of the elapsed time (the job is as
slow as its slowest rank).

Sequence sharding (long contexts with fewer sequences than ranks): every rank
holds a contiguous token range of each sequence (``token_ranges``) and runs
decode + combine on it; one all-gather brings every rank's (o_lat, lse) to
every rank (``gather_partials``) and the library's log-sum-exp merge gives the
whole-sequence result (``sequence_sharded_attend``).

Works with any torch.distributed backend (NCCL on GPUs, gloo for the CPU
tests).
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


# ---------------------------------------------------------------------------
# Sequence sharding
# ---------------------------------------------------------------------------
def token_ranges(lens, world: int, tile: int = 64):
    """Token range [lo, hi) of every sequence held by each rank.

    The sequences' 64-token tiles, concatenated in batch order (T tiles), are
    dealt into ``world`` contiguous runs as the decode deals tiles to its
    workers: rank r takes tiles [r*T // world, (r+1)*T // world).  So every
    token of every sequence is on exactly one rank, each rank's share of a
    sequence is one contiguous range, and the ranks' tile counts differ by at
    most one.  Returns an int64 array [world, B, 2]; hi == lo where a rank
    holds nothing of a sequence."""
    import numpy as np

    lens = np.asarray(lens, dtype=np.int64)
    nt = (np.maximum(lens, 0) + tile - 1) // tile
    pre = np.concatenate([[0], np.cumsum(nt)])
    T = int(pre[-1])
    out = np.zeros((world, lens.size, 2), dtype=np.int64)
    for r in range(world):
        t0, t1 = r * T // world, (r + 1) * T // world
        lo_t = np.clip(t0 - pre[:-1], 0, nt)
        hi_t = np.clip(t1 - pre[:-1], 0, nt)
        out[r, :, 0] = np.minimum(lo_t * tile, lens)
        out[r, :, 1] = np.minimum(hi_t * tile, lens)
    return out


def gather_partials(o_lat, lse, world: int):
    """Every rank's (o_lat [B,H,d_c], lse [B,H]) on every rank, stacked by
    rank: ([world,B,H,d_c], [world,B,H]).  One all-gather per tensor."""
    import torch

    if world <= 1:
        return o_lat.unsqueeze(0), lse.unsqueeze(0)
    import torch.distributed as dist
    o_all = [torch.empty_like(o_lat) for _ in range(world)]
    l_all = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(o_all, o_lat.contiguous())
    dist.all_gather(l_all, lse.contiguous())
    return torch.stack(o_all), torch.stack(l_all)


def sequence_sharded_attend(step, q_nope, q_pe, q_pos, local_cache, local_seqlens, world: int):
    """One attention step over a sequence-sharded cache on this rank.

    ``step`` is a DecodeStep whose dims carry the local cache's capacity;
    ``local_cache`` [B, capacity, R] holds this rank's token range of every
    sequence (rows stored with their global RoPE positions, so slicing needs
    no re-rotation) and ``local_seqlens`` [B] int32 the range lengths; the
    query inputs are the same on every rank (q_pos is the global position).
    Absorb, decode and combine run on the local range, the per-range results
    are all-gathered, merged by the library's log-sum-exp merge and projected
    by W^UV.  Returns step.out [B,H,d_v], the same on every rank."""
    from . import binding as bd

    dims = step.dims
    step.absorb(q_nope, q_pe, q_pos)
    used = bd.decode(dims, step.q_cat, local_cache, local_seqlens, step.scale, step.ws,
                     step.num_splits)
    bd.combine(dims, local_seqlens, step.ws, used, step.o_lat, step.lse)
    if world > 1:   # one rank's range is the whole sequence: nothing to merge
        o_parts, lse_parts = gather_partials(step.o_lat, step.lse, world)
        bd.merge_partials(dims, o_parts, lse_parts, step.o_lat, step.lse)
    bd.out_proj(dims, step.o_lat, step.W_UV, step.out)
    return step.out
