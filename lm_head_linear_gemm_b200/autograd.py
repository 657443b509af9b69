"""``torch.autograd`` drop-in for the fused linear cross-entropy.

    loss = fused_linear_cross_entropy(hidden, lm_head_weight, targets, Vreal=50257, cap=15.0)
    loss.backward()

When a gradient is needed the forward call already forms dX and dW in the same
pass over the logits (the gradient of the mean loss); backward only multiplies
them by the upstream gradient inside the library.  Otherwise the forward keeps
only the per-row log-sum-exp.
"""
from __future__ import annotations

import torch

from . import _abi


class FusedLinearCrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, targets, Vreal, cap, ignore_index, chunk_rows):
        need = ctx.needs_input_grad[0] or ctx.needs_input_grad[1]
        loss, lse, dX, dW, ws = _abi.forward(X, W, targets, Vreal, cap, ignore_index,
                                             want_grads=need, chunk_rows=chunk_rows)
        ctx.meta = (Vreal, cap, ignore_index, chunk_rows)
        if need:
            ctx.save_for_backward(X, W, targets, lse, dX, dW)
        return loss

    @staticmethod
    def backward(ctx, g):
        X, W, targets, lse, dX, dW = ctx.saved_tensors
        Vreal, cap, ignore_index, chunk_rows = ctx.meta
        g = g.detach().to(torch.float32).contiguous()
        _abi.backward(X, W, targets, lse, Vreal, cap, ignore_index, grad_out=g, dX=dX, dW=dW,
                      grads_precomputed=True)
        return (dX if ctx.needs_input_grad[0] else None,
                dW if ctx.needs_input_grad[1] else None, None, None, None, None, None)


def fused_linear_cross_entropy(X, W, targets, Vreal: int, cap: float = 15.0,
                               ignore_index: int = -1, chunk_rows: int = 0):
    """Mean softcapped cross entropy of ``X W^T`` over rows whose target is not ignore_index."""
    return FusedLinearCrossEntropy.apply(X, W, targets, Vreal, cap, ignore_index, chunk_rows)


class RMSNorm(torch.autograd.Function):
    """The model's final RMSNorm in front of the head, in the library's kernels."""

    @staticmethod
    def forward(ctx, H, gamma, eps):
        X, rstd = _abi.rmsnorm_forward(H.contiguous(), gamma.contiguous(), eps)
        ctx.save_for_backward(H, gamma, rstd)
        return X

    @staticmethod
    def backward(ctx, dX):
        H, gamma, rstd = ctx.saved_tensors
        dH, dgamma = _abi.rmsnorm_backward(H, gamma, rstd, dX.contiguous())
        return dH, dgamma, None


def rmsnorm(H, gamma, eps: float = 1e-6):
    """x = h / sqrt(mean(h^2) + eps) * gamma, with a backward into H and gamma."""
    return RMSNorm.apply(H, gamma, eps)
