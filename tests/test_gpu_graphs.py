"""The calls inside a CUDA graph: a forward and a backward captured once and
replayed give the same bits as the eager calls, for the captured inputs and,
after new values are copied into the captured buffers, for those too (the graph
reads the buffers at replay, nothing is baked in but pointers, sizes, alpha and
b).  The lengths are device tensors, so a replay also follows new lengths."""
import math

import numpy as np
import pytest
import torch

import oracle
from padding_aware_sigmoid_b200 import workloads
from tests import _compare as C

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("padding_aware_sigmoid_b200")


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _eager(q, k, v, do, n, alpha, bias):
    o = sa.fwd(q, k, v, n, n, alpha, bias)
    dq, dk, dv = sa.bwd(q, k, v, do, n, n, alpha, bias)
    return o, dq, dk, dv


@pytest.mark.parametrize("D", [64, 128])
def test_forward_backward_replay_from_a_graph(D):
    dev = _dev()
    Z, L, H = 2, 640, 2
    alpha, bias = 1.0 / math.sqrt(D), -math.log(L)
    bufs = [t.to(dev) for t in workloads.random_tensors(Z, L, H, D, 7100 + D, "bf16")]
    n = torch.tensor([640, 333], dtype=torch.int32, device=dev)
    want = _eager(*bufs, n, alpha, bias)
    outs = [torch.empty_like(bufs[0]) for _ in range(4)]

    def body():
        sa.fwd(bufs[0], bufs[1], bufs[2], n, n, alpha, bias, out=outs[0])
        sa.bwd(*bufs, n, n, alpha, bias, dq=outs[1], dk=outs[2], dv=outs[3])

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        body()
    torch.cuda.current_stream(dev).wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        body()
    for t in outs:
        t.zero_()
    g.replay()
    torch.cuda.synchronize(dev)
    assert sa.last_device_status() == 0
    for name, got, ref in zip(("O", "dQ", "dK", "dV"), outs, want):
        assert torch.equal(got, ref), name + " differs between replay and eager call"

    # new values in the captured buffers, and new lengths
    fresh = workloads.random_tensors(Z, L, H, D, 7200 + D, "bf16")
    for b, f in zip(bufs, fresh):
        b.copy_(f.to(dev))
    n.copy_(torch.tensor([129, 640], dtype=torch.int32, device=dev))
    g.replay()
    torch.cuda.synchronize(dev)
    assert sa.last_device_status() == 0
    want = _eager(*bufs, n, alpha, bias)
    for name, got, ref in zip(("O", "dQ", "dK", "dV"), outs, want):
        assert torch.equal(got, ref), name + " differs after new inputs"
    lens = np.array([129, 640], np.int32)
    ro = oracle.fwd(*fresh[:3], lens, lens, alpha, bias)
    C.assert_close(outs[0].float().cpu().numpy(), ro, "bf16", "O replayed on new inputs")
