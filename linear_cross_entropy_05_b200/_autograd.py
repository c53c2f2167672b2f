"""torch.autograd wrapper: mean cross-entropy of E C^T over non-ignored tokens.

The forward keeps only the per-token log-sum-exp and largest logit (2N
floats) for the backward pass, which recomputes the logit tiles on chip; the
N x V logits are never stored.  The largest logits let the gradient filter's
pre-pass prove more token blocks negligible.  The mean reduction and the dtype cast of the gradients are the
caller-side plumbing around the two C-ABI calls.
"""
from __future__ import annotations

import torch

from . import backward as _cce_backward
from . import forward as _cce_forward


class LinearCrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, E, C, y, ignore_index: int, filter_eps: float):
        row_max = torch.empty(E.shape[0], dtype=torch.float32, device=E.device)
        loss, lse = _cce_forward(E.contiguous(), C.contiguous(), y.contiguous(), ignore_index, row_max=row_max)
        keep = y != ignore_index
        n = keep.sum()
        ctx.save_for_backward(E, C, y, lse, row_max, keep, n)
        ctx.ignore_index = ignore_index
        ctx.filter_eps = filter_eps
        return loss.sum() / n

    @staticmethod
    def backward(ctx, g):
        E, C, y, lse, row_max, keep, n = ctx.saved_tensors
        dloss = keep.to(torch.float32) * (g.to(torch.float32) / n.to(torch.float32))
        dE, dC = _cce_backward(E.contiguous(), C.contiguous(), y.contiguous(), lse, dloss.contiguous(),
                               ctx.filter_eps, ctx.ignore_index, row_max=row_max)
        return dE.to(E.dtype), dC.to(C.dtype), None, None, None
