"""Host-side sharding of a padded batch over ranks (one process per GPU).

Every (sample, head) problem of padding-aware sigmoid attention is
independent, so a batch splits over GPUs with no data-path collective: each
rank runs the kernels on its own samples.  With variable lengths the work of
sample z is proportional to n_q(z) * n_k(z) (only valid tiles are computed), so
samples are assigned greedily, longest first, to the least-loaded rank (LPT).
"""
from __future__ import annotations

import numpy as np


def sample_cost(seqlens_q, seqlens_k, block: int = 128) -> np.ndarray:
    """Work of each sample in 128x128 tile pairs (what the kernels compute)."""
    nq = np.asarray(seqlens_q, dtype=np.int64)
    nk = np.asarray(seqlens_k, dtype=np.int64)
    return ((nq + block - 1) // block) * ((nk + block - 1) // block)


def balanced_shards(seqlens_q, seqlens_k, world: int):
    """Sample indices per rank (sorted), balancing tile-pair work by LPT."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = sample_cost(seqlens_q, seqlens_k)
    order = np.argsort(-cost, kind="stable")
    load = np.zeros(world, dtype=np.int64)
    shards = [[] for _ in range(world)]
    for z in order:
        r = int(np.argmin(load))
        shards[r].append(int(z))
        load[r] += int(cost[z])
    return [sorted(s) for s in shards]


def shard_of(seqlens_q, seqlens_k, world: int, rank: int):
    return balanced_shards(seqlens_q, seqlens_k, world)[rank]
