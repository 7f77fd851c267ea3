"""Context parallelism's exchange steps on CPU: world-size-2 gloo ranks each hold a
slice of the sequence, all-gather K and V, compute their queries against every
key and add the dK, dV contributions across ranks, both by the reduce-scatter
on the chunked layout (the route NCCL takes) and by all-reduce and slice.  The
per-rank compute is the fp64 oracle's rectangular route (the GPU kernels do not
run on a CPU host); the reassembled result must equal the oracle on the
unsplit sequence."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from padding_aware_sigmoid_b200 import context_parallel as cp


class _OracleKernels:
    """fwd_rect / bwd_rect with the oracle on CPU tensors (fp32 in and out)."""

    @staticmethod
    def fwd_rect(q, k, v, nq, nk, alpha, bias):
        import oracle
        o = oracle.fwd(q, k, v, nq.numpy(), nk.numpy(), alpha, bias)
        return torch.from_numpy(o.astype(np.float32))

    @staticmethod
    def bwd_rect(q, k, v, dout, nq, nk, alpha, bias):
        import oracle
        g = oracle.bwd(q, k, v, dout, nq.numpy(), nk.numpy(), alpha, bias)
        return tuple(torch.from_numpy(x.astype(np.float32)) for x in g)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q, k, v, do, n, alpha, bias, out, method):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = q.shape[1]
        ls = L // world
        sl = slice(rank * ls, (rank + 1) * ls)
        loc = [torch.from_numpy(np.ascontiguousarray(a[:, sl])) for a in (q, k, v, do)]
        nt = torch.from_numpy(n)
        o = cp.forward(loc[0], loc[1], loc[2], nt, alpha, bias, kernels=_OracleKernels)
        dq, dk, dv = cp.backward(*loc, nt, alpha, bias, kernels=_OracleKernels, method=method)
        out.put((rank, o.numpy(), dq.numpy(), dk.numpy(), dv.numpy()))
    finally:
        dist.destroy_process_group()


def test_local_lengths():
    n = torch.tensor([0, 5, 16, 9, 12], dtype=torch.int32)
    assert cp.local_lengths(n, 0, 2, 16).tolist() == [0, 5, 8, 8, 8]
    assert cp.local_lengths(n, 1, 2, 16).tolist() == [0, 0, 8, 1, 4]
    with pytest.raises(ValueError):
        cp.local_lengths(n, 0, 3, 16)


def test_chunked_layout_round_trip():
    x = torch.arange(2 * 8 * 3 * 4, dtype=torch.float32).reshape(2, 8, 3, 4)
    xt = cp.rows_to_chunks(x)
    for r, chunk in enumerate(xt.chunk(4)):
        # chunk r of the first dimension holds rank r's rows of every sample
        assert torch.equal(cp.chunks_to_rows(chunk), x[:, 2 * r:2 * r + 2])


@pytest.mark.timeout(300)
@pytest.mark.parametrize("method", ["reduce_scatter", "all_reduce"])
def test_two_gloo_ranks_context_parallel(method):
    g = np.random.default_rng(1)
    Z, L, H, D = 3, 16, 2, 8
    q, k, v, do = (g.standard_normal((Z, L, H, D)).astype(np.float32) for _ in range(4))
    n = np.array([16, 11, 6], np.int32)     # one full, one ending in rank 1's slice, one in rank 0's
    alpha, bias = 0.35, -1.2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, k, v, do, n, alpha, bias, out,
                                               method))
             for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, rest) for r, *rest in (out.get(timeout=240) for _ in range(2)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    want_o = oracle.fwd(q, k, v, n, n, alpha, bias)
    want_g = oracle.bwd(q, k, v, do, n, n, alpha, bias)
    got = [np.concatenate([res[r][i] for r in range(2)], axis=1) for i in range(4)]
    for name, a, b in zip(("O", "dQ", "dK", "dV"), got, (want_o,) + tuple(want_g)):
        err = np.abs(a - b).max()
        assert err <= 1e-5 * max(1.0, np.abs(b).max()), (name, err)
