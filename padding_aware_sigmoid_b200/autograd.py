"""Drop-in autograd wrapper: a ``torch.autograd.Function`` whose forward and
backward are the library's kernels (the pages' PyTorch integration,
paper.rainbus.top summary, reproducibility notes; paperlayer.ai summary,
section 2).  The backward recomputes P, so only Q, K, V and the lengths are
saved."""
from __future__ import annotations

import math

import torch


class _SigmoidAttentionFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, seqlens_q, seqlens_k, alpha, bias):
        from . import fwd
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        out = fwd(q, k, v, seqlens_q, seqlens_k, alpha, bias)
        ctx.save_for_backward(q, k, v, seqlens_q, seqlens_k)
        ctx.alpha, ctx.bias = alpha, bias
        return out

    @staticmethod
    def backward(ctx, dout):
        from . import bwd
        q, k, v, nq, nk = ctx.saved_tensors
        dq, dk, dv = bwd(q, k, v, dout.contiguous(), nq, nk, ctx.alpha, ctx.bias)
        return dq, dk, dv, None, None, None, None


class SigmoidAttention(torch.nn.Module):
    """sigma(alpha Q K^T + b) V over padded [Z, L, H, D] batches.

    ``alpha`` defaults to 1/sqrt(D) and ``bias`` to -ln(L) (the pages' b = -log n
    with n the padded length; gist.science summary, section 2.A)."""

    def __init__(self, alpha: float | None = None, bias: float | None = None):
        super().__init__()
        self.alpha, self.bias = alpha, bias

    def forward(self, q, k, v, seqlens_q, seqlens_k=None):
        if seqlens_k is None:
            seqlens_k = seqlens_q
        D, L = q.shape[-1], q.shape[1]
        alpha = 1.0 / math.sqrt(D) if self.alpha is None else self.alpha
        bias = -math.log(L) if self.bias is None else self.bias
        return _SigmoidAttentionFn.apply(q, k, v, seqlens_q, seqlens_k, float(alpha), float(bias))
