"""The N > 1 path on CPU: world-size-2 gloo ranks each take their LPT shard of
a padded batch, compute it (with the fp64 oracle standing in for the GPU
kernels, which need no collective), and the gathered result must equal the
unsharded one; the benchmark's max-over-ranks timing reduction is checked too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from padding_aware_sigmoid_b200 import sharding


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q, k, v, nq, nk, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import bench
        mine = sharding.shard_of(nq, nk, world, rank)
        Z, L, H, D = q.shape
        local = np.zeros((Z, L, H, D))
        if mine:
            idx = np.asarray(mine)
            o = oracle.fwd(q[idx], k[idx], v[idx], nq[idx], nk[idx], 0.3, -1.0)
            local[idx] = o
        t = torch.from_numpy(local)
        dist.all_reduce(t)  # shards are disjoint: the sum reassembles the batch
        # max-over-ranks timing, as bench.py reports it
        m = bench.max_over_ranks(float(rank + 1), world, torch.device("cpu"))
        if rank == 0:
            out.put((t.numpy(), m))
    finally:
        dist.destroy_process_group()


def test_lpt_shards_cover_batch_once():
    nq = np.array([100, 4000, 300, 2500, 16384, 50, 0, 900])
    for world in (1, 2, 3, 5):
        shards = sharding.balanced_shards(nq, nq, world)
        flat = sorted(z for s in shards for z in s)
        assert flat == list(range(len(nq)))
    cost = sharding.sample_cost(nq, nq)
    s2 = sharding.balanced_shards(nq, nq, 2)
    loads = [int(cost[s].sum()) for s in s2]
    assert max(loads) == int(cost.max())  # the 16K sample alone dominates one rank


@pytest.mark.timeout(300)
def test_two_gloo_ranks_reassemble_the_batch():
    g = np.random.default_rng(0)
    Z, L, H, D = 4, 40, 2, 8
    q, k, v = (g.standard_normal((Z, L, H, D)).astype(np.float32) for _ in range(3))
    nq = np.array([40, 7, 23, 0], np.int32)
    nk = np.array([31, 40, 1, 12], np.int32)
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, k, v, nq, nk, out)) for r in range(2)]
    for p in procs:
        p.start()
    got, m = out.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    want = oracle.fwd(q, k, v, nq, nk, 0.3, -1.0)
    assert np.array_equal(got, want)
    assert m == 2.0
