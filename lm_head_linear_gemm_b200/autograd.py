"""``torch.autograd`` drop-ins for the fused linear cross-entropy, the final RMSNorm, and the two
in one call.

    loss = fused_linear_cross_entropy(hidden, lm_head_weight, targets, Vreal=50257, cap=15.0)
    loss.backward()

How the head's gradient is formed depends on what the weight carries:

* plain weight (default): the forward forms dX and dW for g = 1 in the same pass over the
  logits that gives the loss (dW in the weight's dtype, so bf16 for a bf16 head); backward
  multiplies both by the upstream gradient g in place and hands them to autograd, which
  accumulates W.grad across micro-batches in the weight's dtype (bf16 master weights, as the
  pages train).
* ``W.main_grad`` (an fp32 tensor of W's shape, the mixed-precision convention): the library
  adds the gradient into main_grad in fp32 and W.grad is left untouched.  Without a hint the
  forward keeps only the per-row log-sum-exp and backward recomputes the logits with g known
  (8 N d Vpad FLOPs instead of 6).
* ``W.main_grad`` and ``grad_scale=g0``: the forward adds g0 * dW into main_grad in the same
  pass (6 N d Vpad FLOPs), for a training loop that already knows g (e.g. 1/7 when each of 7
  micro-batch losses is divided by 7); backward checks on the host that the upstream gradient
  equals g0 and raises if it does not.

Each backward runs once (``once_differentiable``); a second backward through the same graph
raises instead of scaling the saved gradients twice.
"""
from __future__ import annotations

import torch
from torch.autograd.function import once_differentiable

from . import _abi


class FusedLinearCrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, targets, Vreal, cap, ignore_index, chunk_rows, grad_scale):
        need = ctx.needs_input_grad[0] or ctx.needs_input_grad[1]
        main_grad = getattr(W, "main_grad", None) if ctx.needs_input_grad[1] else None
        ctx.meta = (Vreal, cap, ignore_index, chunk_rows)
        ctx.done = False
        ctx.mode = "none"
        if not need:
            loss, _, _, _, _ = _abi.forward(X, W, targets, Vreal, cap, ignore_index,
                                            chunk_rows=chunk_rows)
            return loss
        if main_grad is not None:
            if main_grad.dtype != torch.float32 or tuple(main_grad.shape) != tuple(W.shape):
                raise TypeError("W.main_grad must be a float32 tensor of W's shape")
            if grad_scale is None:
                # g is not known yet: keep lse, recompute in backward with g
                loss, lse, _, _, _ = _abi.forward(X, W, targets, Vreal, cap, ignore_index,
                                                  chunk_rows=chunk_rows)
                ctx.mode = "recompute"
                ctx.save_for_backward(X, W, targets, lse)
                ctx.main_grad = main_grad
                return loss
            g0 = torch.tensor(float(grad_scale), dtype=torch.float32, device=X.device)
            loss, _, dX, _, _ = _abi.forward(X, W, targets, Vreal, cap, ignore_index,
                                             want_grads=True, dW=main_grad, accumulate_dW=True,
                                             grad_scale=g0, chunk_rows=chunk_rows)
            ctx.mode = "hinted"
            ctx.save_for_backward(dX, g0)
            return loss
        dW_dtype = W.dtype if W.dtype in (torch.float32, torch.bfloat16) else torch.float32
        loss, lse, dX, dW, _ = _abi.forward(X, W, targets, Vreal, cap, ignore_index,
                                            want_grads=True, chunk_rows=chunk_rows,
                                            dW_dtype=dW_dtype)
        ctx.mode = "fused"
        ctx.save_for_backward(X, W, targets, lse, dX, dW)
        return loss

    @staticmethod
    @once_differentiable
    def backward(ctx, g):
        if ctx.done:
            raise RuntimeError("fused_linear_cross_entropy: backward already ran for this graph "
                               "(its gradients were formed in place)")
        ctx.done = True
        Vreal, cap, ignore_index, chunk_rows = ctx.meta
        g = g.detach().to(torch.float32).contiguous()
        wants = ctx.needs_input_grad
        if ctx.mode == "fused":
            X, W, targets, lse, dX, dW = ctx.saved_tensors
            _abi.backward(X, W, targets, lse, Vreal, cap, ignore_index, grad_out=g, dX=dX, dW=dW,
                          grads_precomputed=True)
            return (dX if wants[0] else None, dW if wants[1] else None,
                    None, None, None, None, None, None)
        if ctx.mode == "recompute":
            X, W, targets, lse = ctx.saved_tensors
            dX, _ = _abi.backward(X, W, targets, lse, Vreal, cap, ignore_index, grad_out=g,
                                  dW=ctx.main_grad, accumulate_dW=True, chunk_rows=chunk_rows)
            return (dX if wants[0] else None, None, None, None, None, None, None, None)
        dX, g0 = ctx.saved_tensors                                   # "hinted"
        if not torch.equal(g, g0):
            raise RuntimeError(f"fused_linear_cross_entropy: upstream gradient {g.item()} differs "
                               f"from grad_scale {g0.item()} already applied to W.main_grad")
        return (dX if wants[0] else None, None, None, None, None, None, None, None)


def fused_linear_cross_entropy(X, W, targets, Vreal: int, cap: float = 15.0,
                               ignore_index: int = -1, chunk_rows: int = 0,
                               grad_scale: float | None = None):
    """Mean softcapped cross entropy of ``X W^T`` over rows whose target is not ignore_index.

    ``grad_scale`` only matters when W carries ``main_grad``: it is the upstream gradient the
    caller will back-propagate (the forward then accumulates into main_grad in the same pass)."""
    return FusedLinearCrossEntropy.apply(X, W, targets, Vreal, cap, ignore_index, chunk_rows,
                                         grad_scale)


class FusedRMSNormLinearCrossEntropy(torch.autograd.Function):
    """The model's final RMSNorm and the head in one library call (flce_forward_rmsnorm): the
    forward forms the loss and, for g = 1, the gradients of the rows before the norm, of gamma
    and of the head -- the norm's backward folded into the dX contraction, so dX itself is never
    stored -- and backward multiplies them by the upstream gradient in place."""

    @staticmethod
    def forward(ctx, H, gamma, W, targets, Vreal, cap, ignore_index, eps, chunk_rows):
        ctx.meta = (Vreal, cap, ignore_index)
        ctx.done = False
        if not any(ctx.needs_input_grad[:3]):
            loss, _, _, _, _, _ = _abi.forward_rmsnorm(H, gamma, W, targets, Vreal, cap,
                                                       ignore_index, eps, chunk_rows=chunk_rows)
            return loss
        dW_dtype = W.dtype if W.dtype in (torch.float32, torch.bfloat16) else torch.float32
        loss, _, dH, dgamma, dW, _ = _abi.forward_rmsnorm(
            H, gamma, W, targets, Vreal, cap, ignore_index, eps, want_grads=True,
            chunk_rows=chunk_rows, dW_dtype=dW_dtype)
        ctx.save_for_backward(dH, dgamma, dW)
        return loss

    @staticmethod
    @once_differentiable
    def backward(ctx, g):
        if ctx.done:
            raise RuntimeError("fused_rmsnorm_linear_cross_entropy: backward already ran for this "
                               "graph (its gradients were formed in place)")
        ctx.done = True
        Vreal, cap, ignore_index = ctx.meta
        dH, dgamma, dW = ctx.saved_tensors
        g = g.detach().to(torch.float32).contiguous()
        _abi.scale_grads_rmsnorm(g, dH, dgamma, dW, Vreal, cap, ignore_index)
        wants = ctx.needs_input_grad
        return (dH if wants[0] else None, dgamma if wants[1] else None, dW if wants[2] else None,
                None, None, None, None, None, None)


def fused_rmsnorm_linear_cross_entropy(H, gamma, W, targets, Vreal: int, cap: float = 15.0,
                                       ignore_index: int = -1, eps: float = 1e-6,
                                       chunk_rows: int = 0):
    """Mean softcapped cross entropy of ``rmsnorm(H, gamma) W^T`` over rows whose target is not
    ignore_index, with gradients into H, gamma and W (gamma's gradient is formed in float32 and
    cast to gamma's dtype by autograd).

    The gradients are formed in the forward for g = 1 and scaled by the upstream gradient in
    backward, as in the plain mode of ``fused_linear_cross_entropy``; a ``main_grad`` on W is not
    used here (accumulate into an fp32 buffer with ``_abi.forward_rmsnorm(..., accumulate=True,
    grad_scale=g)`` instead)."""
    return FusedRMSNormLinearCrossEntropy.apply(H, gamma, W, targets, Vreal, cap, ignore_index,
                                                eps, chunk_rows)


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
