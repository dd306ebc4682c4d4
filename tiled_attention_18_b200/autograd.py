"""``attention(q, k, v, ...)``: the library's forward and backward passes as
one differentiable PyTorch operation.

The forward call runs ``flash_attention_forward`` and keeps O and the
per-row LSE; the backward call runs ``flash_attention_backward`` with them
(recomputation: no S x S matrix is stored).  Arguments are those of the two
calls (strided views, Sq != Sk, causal, mask, dropout with seed and offset).
This module only connects the calls to autograd: every step of the
computation runs in the library's kernels.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import flash_attention_backward, flash_attention_forward

# the two calls, looked up at run time (tests substitute stand-ins)
_forward = flash_attention_forward
_backward = flash_attention_backward


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, scale, causal, dropout_p, seed, offset, mask, deterministic):
        o, lse = _forward(q, k, v, scale, causal, dropout_p=dropout_p, seed=seed, offset=offset, mask=mask)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.mask = mask
        ctx.args = (scale, causal, dropout_p, seed, offset, deterministic)
        ctx.mark_non_differentiable(lse)
        return o, lse

    @staticmethod
    def backward(ctx, do, _dlse):
        q, k, v, o, lse = ctx.saved_tensors
        scale, causal, dropout_p, seed, offset, deterministic = ctx.args
        # the kernels read dO row by row: give them a dense one
        do = do.contiguous()
        dq, dk, dv = _backward(q, k, v, o, lse, do, scale, causal, deterministic=deterministic,
                               dropout_p=dropout_p, seed=seed, offset=offset, mask=ctx.mask)
        return dq, dk, dv, None, None, None, None, None, None, None


def attention(q, k, v, scale: Optional[float] = None, causal: bool = False, dropout_p: float = 0.0, seed: int = 0,
              offset: int = 0, mask=None, deterministic: bool = False, return_lse: bool = False):
    """Differentiable attention: softmax(scale * Q K^T [+ masks]) [dropout] V.

    q [B, H, Sq, D], k and v [B, H, Sk, D] (fp16/bf16 CUDA tensors, last
    dimension contiguous).  ``scale`` defaults to 1 / sqrt(D).  Gradients
    flow to q, k and v.  With ``return_lse`` also returns the per-row LSE
    (not differentiable).  Use a new ``offset`` (or ``seed``) for every
    training step that needs fresh dropout decisions.
    """
    if scale is None:
        scale = q.shape[-1] ** -0.5
    o, lse = _Attention.apply(q, k, v, float(scale), bool(causal), float(dropout_p), int(seed), int(offset), mask,
                              bool(deterministic))
    return (o, lse) if return_lse else o
