"""Context parallelism: one sequence split across the ranks of a process group.

Rank r of W holds rows [r Ls, (r + 1) Ls) of Q, K, V and dO (Ls = L / W) of
every sample and head.  Because sigma needs no normalisation over a row
(gist.science summary, section 2.A: each weight is computed on its own), a
query row's output is a plain sum over keys, and a key's dK, dV are plain sums
over queries:

* forward: all-gather K and V, then O for the local queries against every key
  (``fwd_rect``);
* backward: with the gathered K, V, dQ for the local queries, and dK, dV
  contributions of the local queries to every key (``bwd_rect``), which are
  added across ranks by a reduce-scatter (or, on request, an all-reduce and a
  slice) so that each rank ends with the dK, dV rows of its own keys.

The true length n_z of each sample counts from the start of the whole
sequence: rank r's local query length is clamp(n_z - r Ls, 0, Ls), and every
rank sees all n_z keys after the gather.

The compute runs in this package's CUDA kernels; ``kernels`` exists so that the
collective steps can be exercised with another implementation of
``fwd_rect`` / ``bwd_rect`` on hosts without a GPU.  Each rank's dK and dV
contributions come out of the kernels in the input dtype (for bf16 inputs that
is one rounding per rank); they are added across ranks in fp32 and the sum is
cast back to the input dtype.
"""
from __future__ import annotations

import torch


class _CudaKernels:
    @staticmethod
    def fwd_rect(q, k, v, nq, nk, alpha, bias):
        from . import fwd_rect
        return fwd_rect(q, k, v, nq, nk, alpha, bias)

    @staticmethod
    def bwd_rect(q, k, v, dout, nq, nk, alpha, bias):
        from . import bwd_rect
        return bwd_rect(q, k, v, dout, nq, nk, alpha, bias)


def local_lengths(n: torch.Tensor, rank: int, world: int, L: int) -> torch.Tensor:
    """Valid rows of rank ``rank``'s slice: clamp(n - rank L/world, 0, L/world)."""
    if L % world != 0:
        raise ValueError(f"padded length {L} does not split into {world} equal slices")
    ls = L // world
    return (n.to(torch.int64) - rank * ls).clamp(0, ls).to(torch.int32).contiguous()


def local_forward(q_loc, k_all, v_all, n, rank: int, world: int, alpha: float, bias: float,
                  kernels=None):
    """O rows of this rank's query slice against every key (no communication)."""
    kernels = kernels or _CudaKernels
    L = k_all.shape[1]
    nq = local_lengths(n, rank, world, L)
    return kernels.fwd_rect(q_loc, k_all, v_all, nq, n, alpha, bias)


def local_backward(q_loc, k_all, v_all, do_loc, n, rank: int, world: int, alpha: float,
                   bias: float, kernels=None):
    """dQ of this rank's queries, and this rank's dK, dV contributions to every
    key (to be added across ranks); no communication."""
    kernels = kernels or _CudaKernels
    L = k_all.shape[1]
    nq = local_lengths(n, rank, world, L)
    return kernels.bwd_rect(q_loc, k_all, v_all, do_loc, nq, n, alpha, bias)


def _gather_rows(x, group):
    world = torch.distributed.get_world_size(group)
    parts = [torch.empty_like(x) for _ in range(world)]
    torch.distributed.all_gather(parts, x.contiguous(), group=group)
    return torch.cat(parts, dim=1).contiguous()


def rows_to_chunks(x: torch.Tensor) -> torch.Tensor:
    """[Z, L, H, D] -> [L, Z, H, D], contiguous: rank r's rows [r L/W, (r+1) L/W)
    become the r-th of W equal chunks of the first dimension, the layout
    reduce-scatter splits its input by."""
    return x.transpose(0, 1).contiguous()


def chunks_to_rows(x: torch.Tensor) -> torch.Tensor:
    """Inverse of rows_to_chunks on one rank's chunk: [Ls, Z, H, D] -> [Z, Ls, H, D]."""
    return x.transpose(0, 1).contiguous()


def _sum_and_keep_slice(x, group, method: str = "reduce_scatter"):
    """Adds x ([Z, L, H, D], fp32) over the ranks and returns this rank's rows.
    method "reduce_scatter": one reduce-scatter on the chunked layout (each rank
    receives only its rows); "all_reduce": every rank receives the whole sum and
    keeps its rows (for backends without reduce-scatter)."""
    world = torch.distributed.get_world_size(group)
    rank = torch.distributed.get_rank(group)
    ls = x.shape[1] // world
    if method == "reduce_scatter":
        xt = rows_to_chunks(x)
        out = torch.empty((ls,) + xt.shape[1:], dtype=x.dtype, device=x.device)
        torch.distributed.reduce_scatter_tensor(out, xt, group=group)
        return chunks_to_rows(out)
    if method != "all_reduce":
        raise ValueError(f"unknown method {method!r}")
    torch.distributed.all_reduce(x, group=group)
    return x[:, rank * ls:(rank + 1) * ls].contiguous()


def forward(q_loc, k_loc, v_loc, n, alpha: float, bias: float, group=None, kernels=None):
    """Context-parallel forward: returns O for this rank's query slice.
    ``n``: int32 [Z] true lengths of the whole sequences (same on every rank)."""
    rank = torch.distributed.get_rank(group)
    world = torch.distributed.get_world_size(group)
    k_all, v_all = _gather_rows(k_loc, group), _gather_rows(v_loc, group)
    return local_forward(q_loc, k_all, v_all, n, rank, world, alpha, bias, kernels)


def backward(q_loc, k_loc, v_loc, do_loc, n, alpha: float, bias: float, group=None,
             kernels=None, method: str = "reduce_scatter"):
    """Context-parallel backward: (dQ, dK, dV) rows of this rank's slice.
    ``method``: how the dK, dV contributions are added (see _sum_and_keep_slice)."""
    rank = torch.distributed.get_rank(group)
    world = torch.distributed.get_world_size(group)
    k_all, v_all = _gather_rows(k_loc, group), _gather_rows(v_loc, group)
    dq, dk_part, dv_part = local_backward(q_loc, k_all, v_all, do_loc, n, rank, world, alpha,
                                          bias, kernels)
    dk = _sum_and_keep_slice(dk_part.float(), group, method).to(k_loc.dtype)
    dv = _sum_and_keep_slice(dv_part.float(), group, method).to(v_loc.dtype)
    return dq, dk, dv
