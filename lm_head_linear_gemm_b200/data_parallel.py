"""Data-parallel fused linear cross-entropy: one process per GPU, ``torch.distributed``.

The write-ups train the 3.8B model with plain DDP on one 8-GPU node (a gradient all-reduce;
their "distributed strategy" paragraph). Every rank holds the LM head W and its own token
rows. One step here gives exactly the result of a single call on the union of all ranks'
rows:

  1. each rank counts its rows in the loss (library kernel);
  2. all-reduce (sum) of the counts -> global count Nv;
  3. the fused forward+backward normalised by the global Nv (``flce_forward_dp``): the rank's
     share of the mean loss, dX for its rows, its contribution to dW;
  4. all-reduce (sum) of the loss shares and of dW.

With ``buckets > 1`` step 4's dW all-reduce overlaps step 3: the library completes dW in
vocabulary buckets (``flce_forward_dp_bucketed``, the last chunk's gradient contractions run
bucket by bucket, dX with the last one) and records a CUDA event per bucket; each bucket is
all-reduced on a communication stream as soon as its event fires, while the remaining buckets
and dX are still being computed.  DDP overlaps its bucketed gradient all-reduce with the
backward pass in the same way.

With gradient accumulation over micro-batches (``accumulate_dW``, ``grad_scale`` = 1/m for m
micro-batches) the dW all-reduce is needed only once per optimizer step; ``allreduce_dW=False``
skips it for the intermediate micro-batches (as DDP's no_sync does).

``dp_step_rmsnorm`` is the same step with the model's final RMSNorm in front of the head, in one
library call per rank (``flce_forward_rmsnorm_dp``); its parameter gradients are dW and dgamma.
"""
from __future__ import annotations

from . import _abi


class LibraryOps:
    """Device work of a step, all in libflce kernels."""

    def __init__(self):
        self._comm = {}

    def count_valid(self, targets, Vreal, ignore_index):
        import torch
        out = torch.empty(1, dtype=torch.int64, device=targets.device)
        # only N, Vreal and ignore_index matter for the count
        shape = _abi.make_shape(targets.shape[0], 8, max(int(Vreal), 8), int(Vreal), 15.0,
                                ignore_index)
        rc = _abi.lib().flce_count_valid(_abi.ctypes.byref(shape), _abi._ptr(targets),
                                         _abi._ptr(out), _abi._stream(None))
        if rc != _abi.FLCE_OK:
            raise _abi.FlceError(rc, "flce_count_valid")
        return out

    def forward(self, X, W, targets, n_valid_total, Vreal, cap, ignore_index, dW,
                accumulate_dW, workspace, chunk_rows, grad_scale=None):
        return _abi.forward_dp(X, W, targets, n_valid_total, Vreal, cap, ignore_index, True,
                               dW=dW, accumulate_dW=accumulate_dW, workspace=workspace,
                               chunk_rows=chunk_rows, grad_scale=grad_scale)

    def forward_buckets(self, X, W, targets, n_valid_total, Vreal, cap, ignore_index, dW,
                        accumulate_dW, workspace, chunk_rows, n_buckets, grad_scale=None):
        """The forward with dW completed in vocabulary buckets.  Returns (loss, lse, dX, dW,
        [(row slice of dW, CUDA event that marks it final), ...])."""
        import torch
        events = [torch.cuda.Event() for _ in range(n_buckets)]
        loss, lse, dX, dW, bounds, _ = _abi.forward_dp_bucketed(
            X, W, targets, n_valid_total, Vreal, cap, ignore_index, events, dW=dW,
            accumulate_dW=accumulate_dW, workspace=workspace, chunk_rows=chunk_rows,
            grad_scale=grad_scale)
        return loss, lse, dX, dW, [(slice(bounds[b], bounds[b + 1]), events[b])
                                   for b in range(n_buckets)]

    def forward_rmsnorm(self, H, gamma, W, targets, n_valid_total, Vreal, cap, ignore_index, eps,
                        dgamma, dW, accumulate, workspace, chunk_rows, grad_scale=None):
        """The final RMSNorm and the head in one call, normalised by the global count.  Returns
        (loss share, lse, dH, dgamma, dW)."""
        loss, lse, dH, dgamma, dW, _ = _abi.forward_rmsnorm(
            H, gamma, W, targets, Vreal, cap, ignore_index, eps, True, dgamma=dgamma, dW=dW,
            accumulate=accumulate, workspace=workspace, chunk_rows=chunk_rows,
            grad_scale=grad_scale, n_valid_total=n_valid_total)
        return loss, lse, dH, dgamma, dW

    def allreduce_async(self, t, ready, group):
        """All-reduce ``t`` on this device's communication stream once ``ready`` has fired."""
        import torch
        import torch.distributed as dist
        comm = self._comm.get(t.device)
        if comm is None:
            comm = self._comm[t.device] = torch.cuda.Stream(device=t.device)
        comm.wait_event(ready)
        with torch.cuda.stream(comm):
            return dist.all_reduce(t, group=group, async_op=True)


def dp_step(X, W, targets, Vreal: int, cap: float = 15.0, ignore_index: int = -1, *,
            group=None, dW=None, accumulate_dW: bool = False, allreduce_dW: bool = True,
            workspace=None, chunk_rows: int = 0, ops=None, grad_scale=None, buckets: int = 1):
    """One data-parallel fused step.  Returns ``(loss, lse, dX, dW, n_valid_total)`` where loss
    is the mean over all ranks' rows in the loss and dW is summed over ranks (when
    ``allreduce_dW``).  ``buckets > 1`` overlaps the dW all-reduce with the step's last
    gradient contractions (same result)."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    distributed = dist.is_initialized()
    nv = ops.count_valid(targets, Vreal, ignore_index)
    if distributed:
        dist.all_reduce(nv, group=group)
    if distributed and allreduce_dW and buckets > 1:
        loss, lse, dX, dW, pieces = ops.forward_buckets(X, W, targets, nv, Vreal, cap,
                                                        ignore_index, dW, accumulate_dW,
                                                        workspace, chunk_rows, buckets,
                                                        grad_scale)
        works = [ops.allreduce_async(dW[sl], ready, group) for sl, ready in pieces]
        dist.all_reduce(loss, group=group)
        for w in works:
            w.wait()
        return loss, lse, dX, dW, nv
    loss, lse, dX, dW, _ = ops.forward(X, W, targets, nv, Vreal, cap, ignore_index, dW,
                                       accumulate_dW, workspace, chunk_rows, grad_scale)
    if distributed:
        dist.all_reduce(loss, group=group)
        if allreduce_dW:
            dist.all_reduce(dW, group=group)
    return loss, lse, dX, dW, nv


def dp_step_rmsnorm(H, gamma, W, targets, Vreal: int, cap: float = 15.0, ignore_index: int = -1,
                    eps: float = 1e-6, *, group=None, dgamma=None, dW=None,
                    accumulate: bool = False, allreduce_grads: bool = True, workspace=None,
                    chunk_rows: int = 0, ops=None, grad_scale=None):
    """One data-parallel step of the model's final RMSNorm and the head in one call (the norm's
    backward folded into the dX contraction).  Steps 1-2 as in ``dp_step``; step 3 is
    ``flce_forward_rmsnorm_dp``; step 4 all-reduces the loss shares, dW and dgamma (the
    parameters' gradients; dH stays with the rank's rows).  Returns
    ``(loss, lse, dH, dgamma, dW, n_valid_total)``, the same as one call on the union of all
    ranks' rows.  The dW all-reduce follows the call (no vocabulary buckets on this path);
    ``allreduce_grads=False`` skips the parameter all-reduces for intermediate micro-batches."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    distributed = dist.is_initialized()
    nv = ops.count_valid(targets, Vreal, ignore_index)
    if distributed:
        dist.all_reduce(nv, group=group)
    loss, lse, dH, dgamma, dW = ops.forward_rmsnorm(H, gamma, W, targets, nv, Vreal, cap,
                                                    ignore_index, eps, dgamma, dW, accumulate,
                                                    workspace, chunk_rows, grad_scale)
    if distributed:
        dist.all_reduce(loss, group=group)
        if allreduce_grads:
            dist.all_reduce(dW, group=group)
            dist.all_reduce(dgamma, group=group)
    return loss, lse, dH, dgamma, dW, nv
