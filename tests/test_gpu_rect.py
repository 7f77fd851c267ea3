"""GPU parity of the rectangular calls (queries of padded length Lq against keys of
padded length Lk) and of the per-rank compute of context parallelism, emulated
rank after rank on one GPU."""
import math

import numpy as np
import pytest
import torch

import oracle
from padding_aware_sigmoid_b200 import context_parallel as cp
from padding_aware_sigmoid_b200 import workloads
from tests import _compare as C

pytestmark = pytest.mark.gpu

sa = pytest.importorskip("padding_aware_sigmoid_b200")


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _rect_inputs(Z, Lq, Lk, H, D, seed):
    q, do = workloads.random_tensors(Z, Lq, H, D, seed, "bf16", count=2)
    k, v = workloads.random_tensors(Z, Lk, H, D, seed + 1, "bf16", count=2)
    return q, k, v, do


RECT = [
    # Z, Lq, Lk, H, D, n_q, n_k
    (2, 200, 520, 2, 128, (200, 77), (520, 300)),
    (2, 640, 256, 2, 64, (600, 1), (256, 129)),
    (1, 128, 1000, 1, 128, (128,), (999,)),
    (3, 384, 130, 2, 64, (384, 0, 250), (130, 64, 0)),
]


@pytest.mark.parametrize("Z,Lq,Lk,H,D,nq,nk", RECT)
def test_rect_full(Z, Lq, Lk, H, D, nq, nk):
    dev = _dev()
    q, k, v, do = _rect_inputs(Z, Lq, Lk, H, D, seed=5000 + Lq + Lk)
    nq, nk = np.asarray(nq, np.int32), np.asarray(nk, np.int32)
    alpha, bias = 1.0 / math.sqrt(D), -math.log(Lk)
    g = [t.to(dev) for t in (q, k, v, do)]
    nqd, nkd = torch.as_tensor(nq, device=dev), torch.as_tensor(nk, device=dev)
    o = sa.fwd_rect(g[0], g[1], g[2], nqd, nkd, alpha, bias)
    dq, dk, dv = sa.bwd_rect(*g, nqd, nkd, alpha, bias)
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0
    assert o.shape == q.shape and dq.shape == q.shape and dk.shape == k.shape
    ro = oracle.fwd(q, k, v, nq, nk, alpha, bias)
    rdq, rdk, rdv = oracle.bwd(q, k, v, do, nq, nk, alpha, bias)
    for name, got, want, lens in (("O", o, ro, nq), ("dQ", dq, rdq, nq), ("dK", dk, rdk, nk),
                                  ("dV", dv, rdv, nk)):
        a = got.float().cpu().numpy()
        for z in range(Z):
            assert np.all(a[z, lens[z]:] == 0.0), f"{name}: padded rows not zero"
        if np.any(want != 0):
            C.assert_close(a, want, "bf16", name + " (rectangular)")
        else:
            assert np.all(a == 0.0)


def test_rect_with_equal_lengths_is_the_square_call():
    dev = _dev()
    Z, L, H, D = 2, 384, 2, 128
    q, k, v, do = (t.to(dev) for t in workloads.random_tensors(Z, L, H, D, 5100, "bf16"))
    n = torch.tensor([384, 251], dtype=torch.int32, device=dev)
    alpha, b = 1.0 / math.sqrt(D), -math.log(L)
    assert torch.equal(sa.fwd(q, k, v, n, n, alpha, b), sa.fwd_rect(q, k, v, n, n, alpha, b))
    for a, c in zip(sa.bwd(q, k, v, do, n, n, alpha, b), sa.bwd_rect(q, k, v, do, n, n, alpha, b)):
        assert torch.equal(a, c)


def test_context_parallel_ranks_emulated_on_one_gpu():
    """Four ranks' compute, one after the other: query slices of 256 rows against
    every key.  O and dQ rows equal the unsplit call bit for bit (same tiles, same
    summation order); dK, dV summed over the ranks in fp32 meet the parity bar."""
    dev = _dev()
    Z, L, H, D, W = 2, 1024, 2, 128, 4
    q, k, v, do = workloads.random_tensors(Z, L, H, D, 5200, "bf16")
    n = np.array([1024, 700], np.int32)
    alpha, bias = 1.0 / math.sqrt(D), -math.log(L)
    g = [t.to(dev) for t in (q, k, v, do)]
    nd = torch.as_tensor(n, device=dev)
    ls = L // W
    outs, dqs = [], []
    dk = torch.zeros(k.shape, dtype=torch.float32, device=dev)
    dv = torch.zeros(v.shape, dtype=torch.float32, device=dev)
    for r in range(W):
        sl = slice(r * ls, (r + 1) * ls)
        q_r, do_r = g[0][:, sl].contiguous(), g[3][:, sl].contiguous()
        outs.append(cp.local_forward(q_r, g[1], g[2], nd, r, W, alpha, bias))
        dq_r, dk_r, dv_r = cp.local_backward(q_r, g[1], g[2], do_r, nd, r, W, alpha, bias)
        dqs.append(dq_r)
        dk += dk_r.float()
        dv += dv_r.float()
    torch.cuda.synchronize()
    assert sa.last_device_status() == 0
    o_full = sa.fwd(g[0], g[1], g[2], nd, nd, alpha, bias)
    dq_full, _, _ = sa.bwd(*g, nd, nd, alpha, bias)
    assert torch.equal(torch.cat(outs, dim=1), o_full)
    assert torch.equal(torch.cat(dqs, dim=1), dq_full)
    _, rdk, rdv = oracle.bwd(q, k, v, do, n, n, alpha, bias)
    C.assert_close(dk.cpu().numpy(), rdk, "bf16", "dK summed over 4 ranks")
    C.assert_close(dv.cpu().numpy(), rdv, "bf16", "dV summed over 4 ranks")
