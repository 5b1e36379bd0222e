"""The multi-GPU host logic with two ranks over gloo on the CPU: each rank
gets its own shard of sequences (same shapes, its own inputs), the timing
collective returns the slowest rank's time on every rank, and the job's
throughput counts the tokens of all ranks.  No GPU and no data-path
collective are involved."""
import datetime
import os
import socket

import numpy as np

from mla_latent_kv_nope_b200 import dist as mdist
from mla_latent_kv_nope_b200 import inputs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        env = mdist.rank_env()
        w = mdist.shard(inputs.WORKLOADS["ragged_append_bf16"].scaled(B=8, N=1000), env.rank)
        lens = inputs.seqlens(w)
        qn, _ = inputs.query(w.scaled(B=2, H=2))
        mdist.barrier(env.world)
        slowest = mdist.max_over_ranks(1.5 + env.rank, env.world)
        shards = [None] * env.world
        dist.all_gather_object(shards, (lens.tolist(), float(qn.sum()), w.B, w.H))
        out.put((env.rank, env.world, slowest, shards,
                 mdist.job_tokens_per_s(w.B, env.world, 2.0)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_time():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, world, slowest, shards, tps in res:
        assert world == 2
        assert slowest == 2.5                       # max over ranks, on every rank
        assert tps == 8 * 2 / 2e-3                  # both ranks' tokens per step time
        (l0, q0, b0, h0), (l1, q1, b1, h1) = shards
        assert (b0, h0) == (b1, h1) == (8, 64)      # same shapes on every rank
        assert l0 != l1 and q0 != q1                # independent inputs per rank
        assert all(1 <= x <= 1000 for x in l0 + l1)


def test_single_rank_is_identity():
    w = inputs.WORKLOADS["v3_bf16"]
    assert mdist.shard(w, 0) == w
    assert mdist.max_over_ranks(3.25, 1) == 3.25
    assert np.isclose(mdist.job_tokens_per_s(32, 1, 0.5), 64000.0)
