"""Seeded synthetic workloads for padding-aware sigmoid attention.

This module holds the shapes, seeds and length distributions of the five
benchmark/parity workloads and the generators that draw their inputs.  It
contains none of the attention arithmetic, so both the CUDA path's tests and
the fp64 oracle take their inputs from here.

The workloads stand in for the CellxGene single-cell corpus the pages train on
(paper.rainbus.top summary, figure 1: 200 to 16,000 expressed genes per cell),
which is not available here:

1. tiny fp32 parity case: Z=2, H=2, L=128, D=64, n = {128, 77};
2. 2K-context single-cell layer: Z=8, H=12, L=2048, D=64, bf16, n ~ U[256, 2048];
3. 16K kernel benchmark, no padding: Z=2, H=16, L=16384, D=128, bf16, n = L
   (paperlayer.ai summary, section 4: 16K context, head_dim 128);
4. 16K kernel benchmark, 25% padding: Z=4, H=16, L=16384, D=128, bf16,
   n ~ U[8192, 16384] (mean fill 75%; same section's padded benchmark);
5. 8K stress-test shape: Z=4, H=12, L=8192, D=64, bf16, gene-count lengths
   n = round(lognormal(ln 2500, 0.8)) clipped to [200, 8192], Q, K, V scaled
   by 4 (large scores).

Every workload uses alpha = 1/sqrt(D) and b = -ln(L), n_q = n_k = n.  Recipe:
``torch.Generator('cpu').manual_seed(k)`` draws Q, K, V, dO as fp32 N(0, 1) in
that order over the whole padded [Z, L, H, D] extent (padding positions keep
their random values as "garbage"); workload 5 then multiplies Q, K, V by 4;
the result is cast to the workload's dtype.  Lengths come from
``numpy.random.default_rng(k)``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    Z: int
    H: int
    L: int
    D: int
    dtype: str          # "fp32" or "bf16"
    length_rule: str    # "fixed", "uniform", "lognormal"
    fixed_lengths: tuple = ()
    lo: int = 0
    hi: int = 0
    qkv_scale: float = 1.0

    @property
    def seed(self) -> int:
        return self.index

    @property
    def alpha(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def bias(self) -> float:
        return -math.log(self.L)


WORKLOADS = {
    1: Workload(1, "tiny-fp32-L128-d64", 2, 2, 128, 64, "fp32", "fixed", (128, 77)),
    2: Workload(2, "sc-2k-d64-uniform", 8, 12, 2048, 64, "bf16", "uniform", lo=256, hi=2048),
    3: Workload(3, "kernel-16k-d128-nopad", 2, 16, 16384, 128, "bf16", "fixed", (16384, 16384)),
    4: Workload(4, "kernel-16k-d128-pad25", 4, 16, 16384, 128, "bf16", "uniform",
                lo=8192, hi=16384),
    5: Workload(5, "stress-8k-d64-lognormal", 4, 12, 8192, 64, "bf16", "lognormal",
                lo=200, hi=8192, qkv_scale=4.0),
}


def lengths(w: Workload) -> np.ndarray:
    """Per-sample true lengths n (int32[Z]); n_q = n_k = n for every workload."""
    if w.length_rule == "fixed":
        return np.asarray(w.fixed_lengths, dtype=np.int32)
    rng = np.random.default_rng(w.seed)
    if w.length_rule == "uniform":
        return rng.integers(w.lo, w.hi + 1, size=w.Z).astype(np.int32)
    if w.length_rule == "lognormal":
        n = np.rint(rng.lognormal(mean=math.log(2500.0), sigma=0.8, size=w.Z))
        return np.clip(n, w.lo, w.hi).astype(np.int32)
    raise ValueError(w.length_rule)


def _torch_dtype(name: str):
    import torch
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


def random_tensors(Z: int, L: int, H: int, D: int, seed: int, dtype: str = "bf16",
                   qkv_scale: float = 1.0, count: int = 4):
    """Draw ``count`` tensors [Z, L, H, D] ~ N(0, 1) from one CPU generator, in order
    (Q, K, V, dO); Q, K, V are multiplied by ``qkv_scale``; then cast to ``dtype``."""
    import torch
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    out = []
    for t in range(count):
        x = torch.randn((Z, L, H, D), generator=g, dtype=torch.float32)
        if qkv_scale != 1.0 and t < 3:
            x.mul_(qkv_scale)
        out.append(x.to(_torch_dtype(dtype)))
    return out


def make_inputs(w: Workload):
    """CPU tensors and scalars of one workload: dict(q, k, v, dout, seqlens_q, seqlens_k,
    alpha, bias)."""
    q, k, v, do = random_tensors(w.Z, w.L, w.H, w.D, w.seed, w.dtype, w.qkv_scale)
    n = lengths(w)
    return dict(q=q, k=k, v=v, dout=do, seqlens_q=n.copy(), seqlens_k=n.copy(),
                alpha=w.alpha, bias=w.bias)


def fwd_flops_valid(seqlens_q, seqlens_k, H: int, D: int) -> float:
    """Forward FLOPs counted over valid tokens only: 4 D H sum_z n_q(z) n_k(z)
    (two matmuls of 2 D flops per valid query-key pair).  The backward is
    counted as 2.5x this figure (paperlayer.ai summary, appendix A.2, kernel
    benchmarking)."""
    nq = np.asarray(seqlens_q, dtype=np.float64)
    nk = np.asarray(seqlens_k, dtype=np.float64)
    return float(4.0 * D * H * np.sum(nq * nk))


def fwd_flops_padded(Z: int, L: int, H: int, D: int) -> float:
    """Forward FLOPs over the whole padded extent: 4 D H Z L^2."""
    return float(4.0 * D * H * Z * L * L)


BWD_FLOP_FACTOR = 2.5
