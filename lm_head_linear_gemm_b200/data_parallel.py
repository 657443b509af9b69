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

With gradient accumulation over micro-batches (``accumulate_dW``) the dW all-reduce is needed
only once per optimizer step; ``allreduce_dW=False`` skips it for the intermediate
micro-batches (as DDP's no_sync does).
"""
from __future__ import annotations

from . import _abi


class LibraryOps:
    """Device work of a step, all in libflce kernels."""

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
                accumulate_dW, workspace, chunk_rows):
        return _abi.forward_dp(X, W, targets, n_valid_total, Vreal, cap, ignore_index, True,
                               dW=dW, accumulate_dW=accumulate_dW, workspace=workspace,
                               chunk_rows=chunk_rows)


def dp_step(X, W, targets, Vreal: int, cap: float = 15.0, ignore_index: int = -1, *,
            group=None, dW=None, accumulate_dW: bool = False, allreduce_dW: bool = True,
            workspace=None, chunk_rows: int = 0, ops=None):
    """One data-parallel fused step.  Returns ``(loss, lse, dX, dW, n_valid_total)`` where loss
    is the mean over all ranks' rows in the loss and dW is summed over ranks (when
    ``allreduce_dW``)."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    nv = ops.count_valid(targets, Vreal, ignore_index)
    if dist.is_initialized():
        dist.all_reduce(nv, group=group)
    loss, lse, dX, dW, _ = ops.forward(X, W, targets, nv, Vreal, cap, ignore_index, dW,
                                      accumulate_dW, workspace, chunk_rows)
    if dist.is_initialized():
        dist.all_reduce(loss, group=group)
        if allreduce_dW:
            dist.all_reduce(dW, group=group)
    return loss, lse, dX, dW, nv
