"""ctypes binding of ``libflce.so`` (include/flce.h).  Argument marshalling only.

PyTorch provides device memory and the current CUDA stream; every step of the
fused linear cross-entropy runs in the library's kernels.  There is no fallback:
if the library is missing, importing the binding's entry points raises.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("FLCE_LIBRARY") or os.path.join(HERE, "libflce.so")
HEADER_PATH = os.path.join(os.path.dirname(HERE), "include", "flce.h")

FLCE_OK = 0
NOALLOC_SCRATCH_BYTES = 16 << 20      # FLCE_NOALLOC_SCRATCH_BYTES in include/flce.h
DEV_BAD_TARGET = 1
DEV_TIMEOUT = 2
DTYPE_F32 = 0                         # FLCE_DTYPE_F32: fp32 dW
DTYPE_BF16 = 1                        # FLCE_DTYPE_BF16: bf16 dW


class FlceError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


class flce_shape(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int64),
        ("d", ctypes.c_int64),
        ("Vpad", ctypes.c_int64),
        ("Vreal", ctypes.c_int64),
        ("cap", ctypes.c_float),
        ("ignore_index", ctypes.c_int64),
        ("chunk_rows", ctypes.c_int64),
    ]


class flce_kernel_stats(ctypes.Structure):
    _fields_ = [
        ("launches_total", ctypes.c_int64),
        ("gemm_launches", ctypes.c_int64 * 3),
        ("gemm_ms", ctypes.c_double * 3),
        ("gemm_flop", ctypes.c_double * 3),
    ]


GEMM_KINDS = ("logits", "dX+dW", "unused")

_lib = None


def declared_functions(header: str = HEADER_PATH) -> list[str]:
    """Names of the functions include/flce.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flce_[a-z0-9_]+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """Load libflce.so (built in-tree by ``python -m lm_head_linear_gemm_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m lm_head_linear_gemm_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    shp = ctypes.POINTER(flce_shape)
    L.flce_workspace_bytes.argtypes = [shp, ctypes.c_int]
    L.flce_workspace_bytes.restype = ctypes.c_size_t
    I = ctypes.c_int
    L.flce_forward.argtypes = [shp, P, P, P, P, P, I, P, P, P, I, I, P, ctypes.c_size_t, P]
    L.flce_forward.restype = ctypes.c_int
    L.flce_backward.argtypes = [shp, P, P, P, P, P, P, P, I, I, I, P, ctypes.c_size_t, P]
    L.flce_backward.restype = ctypes.c_int
    L.flce_read_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32),
                                   ctypes.POINTER(ctypes.c_int64), P]
    L.flce_read_status.restype = ctypes.c_int
    L.flce_forward_fp8.argtypes = [shp, P, P, P, P, P, P, P, P, P, I, I, P, P, P, I, I, P,
                                   ctypes.c_size_t, P]
    L.flce_forward_fp8.restype = ctypes.c_int
    L.flce_quantize_e4m3.argtypes = [P, ctypes.c_int64, P, P, P]
    L.flce_quantize_e4m3.restype = ctypes.c_int
    L.flce_count_valid.argtypes = [shp, P, P, P]
    L.flce_count_valid.restype = ctypes.c_int
    L.flce_forward_dp.argtypes = [shp, P, P, P, P, P, P, I, P, P, P, I, I, P,
                                  ctypes.c_size_t, P]
    L.flce_forward_dp.restype = ctypes.c_int
    L.flce_forward_dp_bucketed.argtypes = [shp, P, P, P, P, P, P, P, P, P, I, I, I,
                                           ctypes.POINTER(P), ctypes.POINTER(ctypes.c_int64), P,
                                           ctypes.c_size_t, P]
    L.flce_forward_dp_bucketed.restype = ctypes.c_int
    L.flce_forward_noalloc.argtypes = [shp, P, P, P, P, P, P]
    L.flce_forward_noalloc.restype = ctypes.c_int
    L.flce_rmsnorm_forward.argtypes = [P, P, ctypes.c_float, ctypes.c_int64, ctypes.c_int64, P,
                                       P, P]
    L.flce_rmsnorm_forward.restype = ctypes.c_int
    L.flce_rmsnorm_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
    L.flce_rmsnorm_workspace_bytes.restype = ctypes.c_size_t
    L.flce_rmsnorm_backward.argtypes = [P, P, P, P, ctypes.c_int64, ctypes.c_int64, P, P,
                                        ctypes.c_int, P, ctypes.c_size_t, P]
    L.flce_rmsnorm_backward.restype = ctypes.c_int
    L.flce_workspace_bytes_rmsnorm.argtypes = [shp, ctypes.c_int]
    L.flce_workspace_bytes_rmsnorm.restype = ctypes.c_size_t
    L.flce_forward_rmsnorm.argtypes = [shp, P, P, ctypes.c_float, P, P, P, P, I, P, P, P, P, I,
                                       I, P, ctypes.c_size_t, P]
    L.flce_forward_rmsnorm.restype = ctypes.c_int
    L.flce_forward_rmsnorm_dp.argtypes = [shp, P, P, ctypes.c_float, P, P, P, P, P, I, P, P,
                                          P, P, I, I, P, ctypes.c_size_t, P]
    L.flce_forward_rmsnorm_dp.restype = ctypes.c_int
    L.flce_scale_grads_rmsnorm.argtypes = [shp, P, P, P, P, I, P]
    L.flce_scale_grads_rmsnorm.restype = ctypes.c_int
    L.flce_selftest_wait_timeout.argtypes = [P, ctypes.c_uint64, P]
    L.flce_selftest_wait_timeout.restype = ctypes.c_int
    L.flce_check_pair_schedule.argtypes = [ctypes.c_int] * 5 + [
        ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64)]
    L.flce_check_pair_schedule.restype = ctypes.c_int
    L.flce_instrument.argtypes = [ctypes.c_int]
    L.flce_instrument.restype = ctypes.c_int
    L.flce_instrument_read.argtypes = [ctypes.POINTER(flce_kernel_stats)]
    L.flce_instrument_read.restype = ctypes.c_int
    L.flce_status_string.argtypes = [ctypes.c_int]
    L.flce_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(code: int) -> str:
    try:
        return lib().flce_status_string(int(code)).decode()
    except ImportError:
        return f"status {code}"


def make_shape(N: int, d: int, Vpad: int, Vreal: int, cap: float = 15.0,
               ignore_index: int = -1, chunk_rows: int = 0) -> flce_shape:
    return flce_shape(int(N), int(d), int(Vpad), int(Vreal), float(cap), int(ignore_index),
                      int(chunk_rows))


def workspace_bytes(shape: flce_shape, want_grads: bool) -> int:
    return int(lib().flce_workspace_bytes(ctypes.byref(shape), 1 if want_grads else 0))


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def raw_forward(shape, X_ptr, W_ptr, t_ptr, loss_ptr, lse_ptr, want_grads, grad_scale_ptr,
                dX_ptr, dW_ptr, dW_dtype, accumulate_dW, ws_ptr, ws_bytes, stream_handle) -> int:
    """Direct C-ABI call with integer pointers (flce_forward's argument order); returns the
    flce_status code."""
    return lib().flce_forward(ctypes.byref(shape), X_ptr, W_ptr, t_ptr, loss_ptr, lse_ptr,
                              int(want_grads), grad_scale_ptr, dX_ptr, dW_ptr, int(dW_dtype),
                              int(accumulate_dW), ws_ptr, int(ws_bytes), stream_handle)


def raw_forward_noalloc(shape, X_ptr, W_ptr, t_ptr, loss_ptr, lse_ptr, stream_handle) -> int:
    """flce_forward_noalloc: loss and lse with the library's own fixed device scratch (no
    workspace, nothing allocated); returns the flce_status code."""
    return lib().flce_forward_noalloc(ctypes.byref(shape), X_ptr, W_ptr, t_ptr, loss_ptr,
                                      lse_ptr, stream_handle)


def raw_backward(shape, X_ptr, W_ptr, t_ptr, lse_ptr, g_ptr, dX_ptr, dW_ptr, dW_dtype,
                 accumulate_dW, grads_precomputed, ws_ptr, ws_bytes, stream_handle) -> int:
    """Direct C-ABI call of flce_backward (its argument order); returns the flce_status code."""
    return lib().flce_backward(ctypes.byref(shape), X_ptr, W_ptr, t_ptr, lse_ptr, g_ptr, dX_ptr,
                               dW_ptr, int(dW_dtype), int(accumulate_dW), int(grads_precomputed),
                               ws_ptr, int(ws_bytes), stream_handle)


def read_status(workspace, stream=None) -> tuple[int, int]:
    """(device status bits, rows in the loss) of the last call that used ``workspace``;
    ``workspace=None`` reads those of the last ``flce_forward_noalloc`` call on the current
    device."""
    st = ctypes.c_uint32(0)
    nv = ctypes.c_int64(0)
    rc = lib().flce_read_status(_ptr(workspace), ctypes.byref(st), ctypes.byref(nv),
                                _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_read_status")
    return int(st.value), int(nv.value)


def check_pair_schedule(pairs: int, T0: int, c0: int, T1: int, c1: int):
    """Host-side check of the contraction kernels' tile schedule: raises FlceError unless every
    tile of both problems goes to exactly one pair; returns (max, min) per-pair cost."""
    hi, lo = ctypes.c_int64(0), ctypes.c_int64(0)
    rc = lib().flce_check_pair_schedule(int(pairs), int(T0), int(c0), int(T1), int(c1),
                                        ctypes.byref(hi), ctypes.byref(lo))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_check_pair_schedule")
    return hi.value, lo.value


def selftest_wait_timeout(workspace, limit_ns: int, stream=None) -> None:
    """Run the bounded-wait self-test into ``workspace``'s status word (see read_status)."""
    rc = lib().flce_selftest_wait_timeout(_ptr(workspace), int(limit_ns), _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_selftest_wait_timeout")


def instrument(enable: bool) -> None:
    """Start (reset) or stop per-launch event timing of the contraction kernels."""
    lib().flce_instrument(1 if enable else 0)


def instrument_read() -> dict:
    """Totals since the last ``instrument(True)``: launches and per-kind time / FLOPs."""
    st = flce_kernel_stats()
    rc = lib().flce_instrument_read(ctypes.byref(st))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_instrument_read")
    kinds = {}
    for k, name in enumerate(GEMM_KINDS):
        kinds[name] = dict(launches=int(st.gemm_launches[k]), ms=float(st.gemm_ms[k]),
                           flop=float(st.gemm_flop[k]))
    return dict(launches_total=int(st.launches_total), gemm=kinds)


def _check_buffer(t, name, dtype, shape, device):
    """A caller-supplied tensor the library reads or writes through a raw pointer: it must be a
    contiguous CUDA tensor on ``device`` with exactly this dtype and shape (a wrong one would
    let a kernel write past its end)."""
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_scalar(t, name, dtype, device):
    """A one-element device tensor (count, scale, upstream gradient)."""
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype or t.numel() != 1:
        raise TypeError(f"{name} must be a one-element {dtype} tensor")


def _check_workspace(ws, device):
    import torch
    if ws is None:
        return
    if not ws.is_cuda or ws.device != device or ws.dtype != torch.uint8 or ws.dim() != 1 \
            or not ws.is_contiguous():
        raise ValueError(f"workspace must be a contiguous 1-D uint8 CUDA tensor on {device}")


def _dW_type(dW, dW_dtype):
    """(torch dtype, FLCE_DTYPE_* code) of the dW output: the given buffer's type, else
    ``dW_dtype`` (default float32)."""
    import torch
    dt = dW.dtype if dW is not None else (dW_dtype if dW_dtype is not None else torch.float32)
    if dt == torch.float32:
        return torch.float32, DTYPE_F32
    if dt == torch.bfloat16:
        return torch.bfloat16, DTYPE_BF16
    raise TypeError(f"dW must be float32 or bfloat16, got {dt}")


def _grad_scale(grad_scale, device):
    """The upstream-gradient scalar as a one-element float32 device tensor (or None)."""
    import torch
    if grad_scale is None:
        return None
    if not isinstance(grad_scale, torch.Tensor):
        return torch.tensor(float(grad_scale), dtype=torch.float32, device=device)
    _check_scalar(grad_scale, "grad_scale", torch.float32, device)
    return grad_scale


def _check(X, W, targets):
    import torch
    if not (X.is_cuda and W.is_cuda and targets.is_cuda):
        raise ValueError("X, W and targets must be CUDA tensors")
    if not (X.device == W.device == targets.device):
        raise ValueError("X, W and targets must be on the same device")
    if X.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("X and W must be bfloat16")
    if targets.dtype != torch.int64:
        raise TypeError("targets must be int64")
    if X.dim() != 2 or W.dim() != 2 or targets.dim() != 1:
        raise ValueError("expected X [N, d], W [Vpad, d], targets [N]")
    if X.shape[1] != W.shape[1] or X.shape[0] != targets.shape[0]:
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, W {tuple(W.shape)}, "
                         f"targets {tuple(targets.shape)}")
    for name, t in (("X", X), ("W", W), ("targets", targets)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def alloc_workspace(shape: flce_shape, want_grads: bool, device):
    import torch
    nbytes = workspace_bytes(shape, want_grads)
    if nbytes == 0:
        raise FlceError(-1, "flce_workspace_bytes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def forward(X, W, targets, Vreal: int, cap: float = 15.0, ignore_index: int = -1,
            want_grads: bool = False, dX=None, dW=None, accumulate_dW: bool = False,
            workspace=None, chunk_rows: int = 0, stream=None, grad_scale=None, dW_dtype=None):
    """Fused forward.  Returns ``(loss [] fp32, lse [N] fp32, dX, dW, workspace)``;
    dX/dW are None unless ``want_grads``.  With ``want_grads`` the gradients are those of
    ``grad_scale * loss`` (a float or a one-element float32 device tensor; None = 1), and dW is
    float32 unless ``dW`` (or ``dW_dtype``) is bfloat16."""
    import torch
    _check(X, W, targets)
    N, d = X.shape
    dev = X.device
    dw_t, dw_code = _dW_type(dW, dW_dtype)
    if want_grads:
        _check_buffer(dX, "dX", torch.bfloat16, X.shape, dev)
        _check_buffer(dW, "dW", dw_t, W.shape, dev)
        grad_scale = _grad_scale(grad_scale, dev)
    _check_workspace(workspace, dev)
    shape = make_shape(N, d, W.shape[0], Vreal, cap, ignore_index, chunk_rows)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse = torch.empty(max(N, 1), dtype=torch.float32, device=dev)[:N]
    if want_grads:
        if dX is None:
            dX = torch.empty_like(X)
        if dW is None:
            dW = torch.empty(W.shape, dtype=dw_t, device=dev)
    if workspace is None:
        workspace = alloc_workspace(shape, want_grads, dev)
    rc = raw_forward(shape, _ptr(X), _ptr(W), _ptr(targets), _ptr(loss), _ptr(lse),
                     want_grads, _ptr(grad_scale) if want_grads else None,
                     _ptr(dX) if want_grads else None, _ptr(dW) if want_grads else None,
                     dw_code, accumulate_dW, _ptr(workspace), workspace.numel(), _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_forward")
    return loss, lse, (dX if want_grads else None), (dW if want_grads else None), workspace


def forward_dp(X, W, targets, n_valid_total, Vreal: int, cap: float = 15.0,
               ignore_index: int = -1, want_grads: bool = True, dX=None, dW=None,
               accumulate_dW: bool = False, workspace=None, chunk_rows: int = 0, stream=None,
               grad_scale=None, dW_dtype=None):
    """flce_forward normalised by a device int64 count of rows in the loss over all
    data-parallel ranks.  Returns (loss share, lse, dX, dW, workspace)."""
    import torch
    _check(X, W, targets)
    N, d = X.shape
    dev = X.device
    if n_valid_total is None:
        raise TypeError("n_valid_total must be a CUDA int64 tensor")
    _check_scalar(n_valid_total, "n_valid_total", torch.int64, dev)
    dw_t, dw_code = _dW_type(dW, dW_dtype)
    if want_grads:
        _check_buffer(dX, "dX", torch.bfloat16, X.shape, dev)
        _check_buffer(dW, "dW", dw_t, W.shape, dev)
        grad_scale = _grad_scale(grad_scale, dev)
    _check_workspace(workspace, dev)
    shape = make_shape(N, d, W.shape[0], Vreal, cap, ignore_index, chunk_rows)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse = torch.empty(max(N, 1), dtype=torch.float32, device=dev)[:N]
    if want_grads:
        if dX is None:
            dX = torch.empty_like(X)
        if dW is None:
            dW = torch.empty(W.shape, dtype=dw_t, device=dev)
    if workspace is None:
        workspace = alloc_workspace(shape, want_grads, dev)
    rc = lib().flce_forward_dp(ctypes.byref(shape), _ptr(X), _ptr(W), _ptr(targets),
                               _ptr(n_valid_total), _ptr(loss), _ptr(lse),
                               1 if want_grads else 0,
                               _ptr(grad_scale) if want_grads else None,
                               _ptr(dX) if want_grads else None,
                               _ptr(dW) if want_grads else None, dw_code, int(accumulate_dW),
                               _ptr(workspace), workspace.numel(), _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_forward_dp")
    return loss, lse, (dX if want_grads else None), (dW if want_grads else None), workspace


def forward_dp_bucketed(X, W, targets, n_valid_total, Vreal: int, cap: float, ignore_index: int,
                        events, dX=None, dW=None, accumulate_dW: bool = False, workspace=None,
                        chunk_rows: int = 0, stream=None, grad_scale=None, dW_dtype=None):
    """forward_dp with gradients whose dW becomes final in len(events) vocabulary buckets:
    the library records ``events[b]`` (torch.cuda.Event) on the stream once dW rows
    ``bounds[b]:bounds[b + 1]`` are complete.  Returns (loss share, lse, dX, dW, bounds,
    workspace)."""
    import torch
    _check(X, W, targets)
    N, d = X.shape
    dev = X.device
    if n_valid_total is None:
        raise TypeError("n_valid_total must be a CUDA int64 tensor")
    _check_scalar(n_valid_total, "n_valid_total", torch.int64, dev)
    dw_t, dw_code = _dW_type(dW, dW_dtype)
    _check_buffer(dX, "dX", torch.bfloat16, X.shape, dev)
    _check_buffer(dW, "dW", dw_t, W.shape, dev)
    grad_scale = _grad_scale(grad_scale, dev)
    _check_workspace(workspace, dev)
    n = len(events)
    st = _stream(stream)
    for ev in events:                       # torch creates the CUDA event on first record
        if not ev.cuda_event:
            ev.record(torch.cuda.current_stream(dev) if stream is None else stream)
    handles = (ctypes.c_void_p * n)(*[ctypes.c_void_p(ev.cuda_event) for ev in events])
    bounds = (ctypes.c_int64 * (n + 1))()
    shape = make_shape(N, d, W.shape[0], Vreal, cap, ignore_index, chunk_rows)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse = torch.empty(max(N, 1), dtype=torch.float32, device=dev)[:N]
    if dX is None:
        dX = torch.empty_like(X)
    if dW is None:
        dW = torch.empty(W.shape, dtype=dw_t, device=dev)
    if workspace is None:
        workspace = alloc_workspace(shape, True, dev)
    rc = lib().flce_forward_dp_bucketed(ctypes.byref(shape), _ptr(X), _ptr(W), _ptr(targets),
                                        _ptr(n_valid_total), _ptr(loss), _ptr(lse),
                                        _ptr(grad_scale), _ptr(dX), _ptr(dW), dw_code,
                                        int(accumulate_dW), n, handles, bounds, _ptr(workspace),
                                        workspace.numel(), st)
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_forward_dp_bucketed")
    return loss, lse, dX, dW, [int(b) for b in bounds], workspace


def rmsnorm_forward(H, gamma, eps: float = 1e-6, X=None, rstd=None, stream=None):
    """x = h * rstd * gamma (bf16), rstd = 1/sqrt(mean(h^2) + eps) (fp32).  Returns (x, rstd)."""
    import torch
    if not H.is_cuda or H.dim() != 2:
        raise ValueError("H must be a 2-D CUDA tensor [N, d]")
    N, d = H.shape
    dev = H.device
    _check_buffer(H, "H", torch.bfloat16, (N, d), dev)
    _check_buffer(gamma, "gamma", torch.bfloat16, (d,), dev)
    _check_buffer(X, "X", torch.bfloat16, (N, d), dev)
    _check_buffer(rstd, "rstd", torch.float32, (N,), dev)
    if X is None:
        X = torch.empty_like(H)
    if rstd is None:
        rstd = torch.empty(max(N, 1), dtype=torch.float32, device=H.device)[:N]
    rc = lib().flce_rmsnorm_forward(_ptr(H), _ptr(gamma), float(eps), N, d, _ptr(X), _ptr(rstd),
                                    _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_rmsnorm_forward")
    return X, rstd


def forward_rmsnorm(H, gamma, W, targets, Vreal: int, cap: float = 15.0, ignore_index: int = -1,
                    eps: float = 1e-6, want_grads: bool = False, dH=None, dgamma=None, dW=None,
                    accumulate: bool = False, workspace=None, chunk_rows: int = 0, stream=None,
                    grad_scale=None, dW_dtype=None, n_valid_total=None):
    """The final RMSNorm and the head in one call (flce_forward_rmsnorm).  Returns
    ``(loss, lse, dH, dgamma, dW, workspace)``; the gradients (None unless ``want_grads``) are
    those of ``grad_scale * loss`` with respect to the rows before the norm, its gamma and the
    head; ``accumulate`` adds into dgamma and dW.  With ``n_valid_total`` (a one-element int64
    device tensor: the rows in the loss over all data-parallel ranks) the call is one rank's
    share (flce_forward_rmsnorm_dp)."""
    import torch
    _check(H, W, targets)
    N, d = H.shape
    dev = H.device
    _check_buffer(gamma, "gamma", torch.bfloat16, (d,), dev)
    if gamma is None:
        raise TypeError("gamma must be a bfloat16 CUDA tensor [d]")
    _check_scalar(n_valid_total, "n_valid_total", torch.int64, dev)
    dw_t, dw_code = _dW_type(dW, dW_dtype)
    if want_grads:
        _check_buffer(dH, "dH", torch.bfloat16, H.shape, dev)
        _check_buffer(dgamma, "dgamma", torch.float32, (d,), dev)
        _check_buffer(dW, "dW", dw_t, W.shape, dev)
        grad_scale = _grad_scale(grad_scale, dev)
    _check_workspace(workspace, dev)
    shape = make_shape(N, d, W.shape[0], Vreal, cap, ignore_index, chunk_rows)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse = torch.empty(max(N, 1), dtype=torch.float32, device=dev)[:N]
    if want_grads:
        if dH is None:
            dH = torch.empty_like(H)
        if dgamma is None:
            dgamma = torch.empty(d, dtype=torch.float32, device=dev)
        if dW is None:
            dW = torch.empty(W.shape, dtype=dw_t, device=dev)
    if workspace is None:
        nbytes = int(lib().flce_workspace_bytes_rmsnorm(ctypes.byref(shape), int(want_grads)))
        if nbytes == 0:
            raise FlceError(-1, "flce_workspace_bytes_rmsnorm")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    g = want_grads
    head = (ctypes.byref(shape), _ptr(H), _ptr(gamma), float(eps), _ptr(W), _ptr(targets))
    tail = (_ptr(loss), _ptr(lse), int(g), _ptr(grad_scale) if g else None,
            _ptr(dH) if g else None, _ptr(dgamma) if g else None, _ptr(dW) if g else None,
            dw_code, int(accumulate), _ptr(workspace), workspace.numel(), _stream(stream))
    if n_valid_total is None:
        rc, name = lib().flce_forward_rmsnorm(*head, *tail), "flce_forward_rmsnorm"
    else:
        rc = lib().flce_forward_rmsnorm_dp(*head, _ptr(n_valid_total), *tail)
        name = "flce_forward_rmsnorm_dp"
    if rc != FLCE_OK:
        raise FlceError(rc, name)
    if not g:
        return loss, lse, None, None, None, workspace
    return loss, lse, dH, dgamma, dW, workspace


def scale_grads_rmsnorm(grad_out, dH, dgamma, dW, Vreal: int, cap: float = 15.0,
                        ignore_index: int = -1, stream=None):
    """dH, dgamma, dW *= grad_out (a one-element float32 device tensor) in place."""
    import torch
    N, d = dH.shape
    dev = dH.device
    _check_scalar(grad_out, "grad_out", torch.float32, dev)
    _check_buffer(dH, "dH", torch.bfloat16, (N, d), dev)
    _check_buffer(dgamma, "dgamma", torch.float32, (d,), dev)
    dw_t, dw_code = _dW_type(dW, None)
    _check_buffer(dW, "dW", dw_t, (dW.shape[0], d), dev)
    shape = make_shape(N, d, dW.shape[0], Vreal, cap, ignore_index, 0)
    rc = lib().flce_scale_grads_rmsnorm(ctypes.byref(shape), _ptr(grad_out), _ptr(dH),
                                        _ptr(dgamma), _ptr(dW), dw_code, _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_scale_grads_rmsnorm")


def rmsnorm_backward(H, gamma, rstd, dX, dH=None, dgamma=None, accumulate_dgamma: bool = False,
                     stream=None):
    """Chain rule through the RMSNorm for dX = dL/dx.  Returns (dH bf16, dgamma fp32)."""
    import torch
    if not H.is_cuda or H.dim() != 2:
        raise ValueError("H must be a 2-D CUDA tensor [N, d]")
    N, d = H.shape
    dev = H.device
    _check_buffer(H, "H", torch.bfloat16, (N, d), dev)
    _check_buffer(gamma, "gamma", torch.bfloat16, (d,), dev)
    _check_buffer(rstd, "rstd", torch.float32, (N,), dev)
    _check_buffer(dX, "dX", torch.bfloat16, (N, d), dev)
    _check_buffer(dH, "dH", torch.bfloat16, (N, d), dev)
    _check_buffer(dgamma, "dgamma", torch.float32, (d,), dev)
    if dH is None:
        dH = torch.empty_like(H)
    if dgamma is None:
        dgamma = torch.empty(d, dtype=torch.float32, device=H.device)
    nbytes = int(lib().flce_rmsnorm_workspace_bytes(N, d))
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=H.device)
    rc = lib().flce_rmsnorm_backward(_ptr(H), _ptr(gamma), _ptr(rstd), _ptr(dX), N, d, _ptr(dH),
                                     _ptr(dgamma), int(accumulate_dgamma), _ptr(ws), ws.numel(),
                                     _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_rmsnorm_backward")
    return dH, dgamma


def quantize_e4m3(x, out=None, scale=None, stream=None):
    """Tensorwise e4m3 quantisation of a bf16 CUDA tensor: returns (uint8 codes, fp32 scale)
    with x ~ codes.view(float8_e4m3fn) * scale."""
    import torch
    if not x.is_cuda or x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise TypeError("x must be a contiguous bf16 CUDA tensor")
    _check_buffer(out, "out", torch.uint8, x.shape, x.device)
    _check_scalar(scale, "scale", torch.float32, x.device)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((), dtype=torch.float32, device=x.device)
    rc = lib().flce_quantize_e4m3(_ptr(x), x.numel(), _ptr(out), _ptr(scale), _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_quantize_e4m3")
    return out, scale


def forward_fp8(X8, W8, scale_x, scale_w, X, W, targets, Vreal: int, cap: float = 15.0,
                ignore_index: int = -1, want_grads: bool = False, dX=None, dW=None,
                accumulate_dW: bool = False, workspace=None, chunk_rows: int = 0, stream=None,
                grad_scale=None, dW_dtype=None, grad_fp8: bool = False):
    """Fused forward with e4m3 logits operands (uint8 codes + fp32 device scales).  The
    gradient contractions use the bf16 copies X/W, or, with ``grad_fp8``, an e5m2 gradient and
    the e4m3 operands (X/W may then be None).  Returns (loss, lse, dX, dW, workspace)."""
    import torch
    for name, t in (("X8", X8), ("W8", W8)):
        if not t.is_cuda or t.dtype not in (torch.uint8, getattr(torch, "float8_e4m3fn", None)):
            raise TypeError(f"{name} must be a CUDA uint8 / float8_e4m3fn tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if X8.dim() != 2 or W8.dim() != 2 or X8.shape[1] != W8.shape[1]:
        raise ValueError(f"expected X8 [N, d], W8 [Vpad, d]; got {tuple(X8.shape)}, "
                         f"{tuple(W8.shape)}")
    N, d = X8.shape
    dev = X8.device
    if W8.device != dev:
        raise ValueError("X8 and W8 must be on the same device")
    _check_scalar(scale_x, "scale_x", torch.float32, dev)
    _check_scalar(scale_w, "scale_w", torch.float32, dev)
    if scale_x is None or scale_w is None:
        raise TypeError("scale_x and scale_w must be one-element float32 CUDA tensors")
    _check_buffer(targets, "targets", torch.int64, (N,), dev)
    dw_t, dw_code = _dW_type(dW, dW_dtype)
    if want_grads:
        if not grad_fp8:
            _check(X, W, targets)
        _check_buffer(X, "X", torch.bfloat16, (N, d), dev)
        _check_buffer(W, "W", torch.bfloat16, tuple(W8.shape), dev)
        _check_buffer(dX, "dX", torch.bfloat16, (N, d), dev)
        _check_buffer(dW, "dW", dw_t, tuple(W8.shape), dev)
        grad_scale = _grad_scale(grad_scale, dev)
    _check_workspace(workspace, dev)
    shape = make_shape(N, d, W8.shape[0], Vreal, cap, ignore_index, chunk_rows)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse = torch.empty(max(N, 1), dtype=torch.float32, device=dev)[:N]
    if want_grads:
        if dX is None:
            dX = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
        if dW is None:
            dW = torch.empty(tuple(W8.shape), dtype=dw_t, device=dev)
    if workspace is None:
        workspace = alloc_workspace(shape, want_grads, dev)
    rc = lib().flce_forward_fp8(ctypes.byref(shape), _ptr(X8), _ptr(W8), _ptr(scale_x),
                                _ptr(scale_w), _ptr(X), _ptr(W), _ptr(targets), _ptr(loss),
                                _ptr(lse), 1 if want_grads else 0, 1 if grad_fp8 else 0,
                                _ptr(grad_scale) if want_grads else None,
                                _ptr(dX) if want_grads else None,
                                _ptr(dW) if want_grads else None, dw_code, int(accumulate_dW),
                                _ptr(workspace), workspace.numel(), _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_forward_fp8")
    return loss, lse, (dX if want_grads else None), (dW if want_grads else None), workspace


def backward(X, W, targets, lse, Vreal: int, cap: float = 15.0, ignore_index: int = -1,
             grad_out=None, dX=None, dW=None, accumulate_dW: bool = False,
             grads_precomputed: bool = False, workspace=None, chunk_rows: int = 0, stream=None,
             dW_dtype=None):
    """Backward.  Returns ``(dX bf16 [N, d], dW [Vpad, d])``; dW is float32 unless ``dW`` (or
    ``dW_dtype``) is bfloat16."""
    import torch
    _check(X, W, targets)
    N, d = X.shape
    dev = X.device
    dw_t, dw_code = _dW_type(dW, dW_dtype)
    _check_buffer(lse, "lse", torch.float32, (N,), dev)
    _check_buffer(dX, "dX", torch.bfloat16, X.shape, dev)
    _check_buffer(dW, "dW", dw_t, W.shape, dev)
    _check_scalar(grad_out, "grad_out", torch.float32, dev)
    _check_workspace(workspace, dev)
    shape = make_shape(N, d, W.shape[0], Vreal, cap, ignore_index, chunk_rows)
    if dX is None:
        dX = torch.empty_like(X)
    if dW is None:
        dW = torch.empty(W.shape, dtype=dw_t, device=dev)
    if workspace is None and not grads_precomputed:
        workspace = alloc_workspace(shape, True, dev)
    rc = raw_backward(shape, _ptr(X), _ptr(W), _ptr(targets), _ptr(lse), _ptr(grad_out),
                      _ptr(dX), _ptr(dW), dw_code, accumulate_dW, grads_precomputed,
                      _ptr(workspace), 0 if workspace is None else workspace.numel(),
                      _stream(stream))
    if rc != FLCE_OK:
        raise FlceError(rc, "flce_backward")
    return dX, dW
