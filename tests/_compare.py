"""Tolerances and row sampling shared by the GPU parity tests.

Tolerance (fixed before any kernel ran): per output tensor, over the valid
rows compared,
  bf16 path: max|x - ref| <= 2e-2 * max|ref|  and  sum|x - ref| / sum|ref| <= 5e-3
  fp32 path: max|x - ref| <= 1e-4 * max|ref|
and every padded row (query rows >= n_q for O and dQ, key rows >= n_k for dK
and dV) must be exactly zero.  Element-wise relative error is not used: it is
undefined where the reference is zero.
"""
from __future__ import annotations

import numpy as np

BF16_MAX_REL = 2e-2
BF16_L1_REL = 5e-3
FP32_MAX_REL = 1e-4


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = np.abs(got - ref)
    scale = max(float(np.max(np.abs(ref))), 1e-30)
    l1 = float(np.sum(diff)) / max(float(np.sum(np.abs(ref))), 1e-30)
    return float(np.max(diff)) / scale, l1


def assert_close(got, ref, dtype: str, what: str):
    max_rel, l1 = errors(got, ref)
    if dtype == "fp32":
        assert max_rel <= FP32_MAX_REL, f"{what}: max-abs/max|ref| = {max_rel:.3e} > {FP32_MAX_REL}"
    else:
        assert max_rel <= BF16_MAX_REL, f"{what}: max-abs/max|ref| = {max_rel:.3e} > {BF16_MAX_REL}"
        assert l1 <= BF16_L1_REL, f"{what}: L1 relative error {l1:.3e} > {BF16_L1_REL}"
    return max_rel, l1


def valid_row_mask(items: np.ndarray, lengths) -> np.ndarray:
    lengths = np.asarray(lengths)
    return items[:, 2] < lengths[items[:, 0]]


def sample_items(Z: int, L: int, H: int, seqlens, per_sample: int, seed: int) -> np.ndarray:
    """(z, h, row) triples: every length boundary row (0, n-1, n, n+1, L-1) plus
    `per_sample` random rows per sample, heads drawn at random."""
    g = np.random.default_rng(seed)
    out = []
    for z in range(Z):
        n = int(seqlens[z])
        rows = {0, L - 1, n - 1, n, n + 1, n - 128, n + 127}
        rows.update(int(r) for r in g.integers(0, L, size=per_sample))
        for r in sorted(x for x in rows if 0 <= x < L):
            out.append((z, int(g.integers(0, H)), r))
    return np.asarray(out, dtype=np.int64)


def gather_rows(t, items: np.ndarray) -> np.ndarray:
    """Rows [n, D] of a [Z, L, H, D] tensor (torch, any device) as float64."""
    import torch
    z = torch.as_tensor(items[:, 0], device=t.device)
    h = torch.as_tensor(items[:, 1], device=t.device)
    r = torch.as_tensor(items[:, 2], device=t.device)
    return t[z, r, h].float().cpu().numpy().astype(np.float64)
