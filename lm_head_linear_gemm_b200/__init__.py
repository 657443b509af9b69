"""Fused LM-head linear + softcapped cross-entropy for B200 (sm_100a).

The compute path is the C-ABI library ``libflce.so`` (include/flce.h), built in-tree
by ``python -m lm_head_linear_gemm_b200.build``; this package only marshals
arguments to it.  Entry points raise if the library is missing: there is no
fallback implementation.
"""
from ._abi import (DEV_BAD_TARGET, DEV_TIMEOUT, FlceError, alloc_workspace, backward,
                   declared_functions, forward, forward_dp, forward_dp_bucketed, forward_fp8,
                   forward_rmsnorm, instrument, instrument_read, lib, make_shape, raw_backward,
                   raw_forward, quantize_e4m3, raw_forward_noalloc, read_status, rmsnorm_backward,
                   rmsnorm_forward, scale_grads_rmsnorm, selftest_wait_timeout, status_string,
                   workspace_bytes)
from .autograd import (FusedLinearCrossEntropy, FusedRMSNormLinearCrossEntropy, RMSNorm,
                       fused_linear_cross_entropy, fused_rmsnorm_linear_cross_entropy, rmsnorm)
from . import data_parallel
from .data_parallel import dp_step, dp_step_rmsnorm

__all__ = [
    "DEV_BAD_TARGET", "DEV_TIMEOUT", "FlceError", "alloc_workspace", "backward",
    "declared_functions", "forward", "forward_dp", "forward_dp_bucketed", "forward_fp8",
    "forward_rmsnorm", "instrument", "instrument_read", "lib", "make_shape", "raw_backward",
    "raw_forward", "quantize_e4m3", "raw_forward_noalloc", "read_status", "rmsnorm_backward",
    "rmsnorm_forward", "scale_grads_rmsnorm", "selftest_wait_timeout", "status_string",
    "workspace_bytes", "FusedLinearCrossEntropy", "FusedRMSNormLinearCrossEntropy",
    "fused_linear_cross_entropy", "fused_rmsnorm_linear_cross_entropy", "dp_step",
    "dp_step_rmsnorm", "RMSNorm",
    "rmsnorm",
]
