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


class _SigmoidAttentionBiasFn(torch.autograd.Function):
    """As _SigmoidAttentionFn with one bias per sample (float32 [Z] tensor); its
    gradient is db_z = sum over heads and valid (i, j) of dS_ij."""

    @staticmethod
    def forward(ctx, q, k, v, seqlens_q, seqlens_k, alpha, bias_z):
        from . import fwd_bias
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        bias_z = bias_z.detach().to(torch.float32).contiguous()
        out = fwd_bias(q, k, v, seqlens_q, seqlens_k, alpha, bias_z)
        ctx.save_for_backward(q, k, v, seqlens_q, seqlens_k, bias_z)
        ctx.alpha = alpha
        return out

    @staticmethod
    def backward(ctx, dout):
        from . import bwd_bias
        q, k, v, nq, nk, bias_z = ctx.saved_tensors
        dq, dk, dv, db = bwd_bias(q, k, v, dout.contiguous(), nq, nk, ctx.alpha, bias_z,
                                  want_dbias=ctx.needs_input_grad[6])
        return dq, dk, dv, None, None, None, db


class SigmoidAttention(torch.nn.Module):
    """sigma(alpha Q K^T + b) V over padded [Z, L, H, D] batches.

    ``alpha`` defaults to 1/sqrt(D).  The bias follows the pages' b = -log n
    (paperlayer.ai summary, section 3; gist.science summary, section 2.A):

    * default: one scalar, ``bias`` or -ln(L) with n the padded length;
    * ``per_sample_bias=True``: b_z = -ln n_k(z), each sample's true length
      (computed on the device by the library, ``log_length_bias``);
    * ``learnable_bias=True``: a scalar parameter trained through
      db = sum_z db_z, created here with the initial value ``bias``, or -ln
      ``max_len`` (the padded length the module will see) when ``bias`` is not
      given, so that an optimiser built from ``parameters()`` before the first
      call already holds it."""

    def __init__(self, alpha: float | None = None, bias: float | None = None,
                 per_sample_bias: bool = False, learnable_bias: bool = False,
                 max_len: int | None = None):
        super().__init__()
        if per_sample_bias and learnable_bias:
            raise ValueError("choose per_sample_bias or learnable_bias, not both")
        self.alpha, self.bias = alpha, bias
        self.per_sample_bias = per_sample_bias
        self.learnable_bias = learnable_bias
        self.b = None
        if learnable_bias:
            if bias is None and max_len is None:
                raise ValueError("learnable_bias needs an initial value: give bias, or max_len "
                                 "for b = -ln(max_len)")
            init = float(bias) if bias is not None else -math.log(max_len)
            self.b = torch.nn.Parameter(torch.tensor(init))

    def forward(self, q, k, v, seqlens_q, seqlens_k=None):
        if seqlens_k is None:
            seqlens_k = seqlens_q
        Z, L, D = q.shape[0], q.shape[1], q.shape[-1]
        alpha = float(1.0 / math.sqrt(D) if self.alpha is None else self.alpha)
        if self.per_sample_bias:
            from . import log_length_bias
            bias_z = log_length_bias(seqlens_k)
            return _SigmoidAttentionBiasFn.apply(q, k, v, seqlens_q, seqlens_k, alpha, bias_z)
        if self.learnable_bias:
            bias_z = self.b.to(device=q.device, dtype=torch.float32).expand(Z)
            return _SigmoidAttentionBiasFn.apply(q, k, v, seqlens_q, seqlens_k, alpha, bias_z)
        bias = -math.log(L) if self.bias is None else self.bias
        return _SigmoidAttentionFn.apply(q, k, v, seqlens_q, seqlens_k, alpha, float(bias))
