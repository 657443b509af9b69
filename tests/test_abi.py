"""Host-side checks of the C-ABI library: it loads without a GPU, exports every
function include/flce.h declares, sizes its scratch without any N x Vpad term, and
rejects bad arguments on the host before anything is launched."""
import ctypes
import os
import subprocess

import pytest

import lm_head_linear_gemm_b200 as flce
from lm_head_linear_gemm_b200 import _abi
from lm_head_linear_gemm_b200 import build as flce_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    flce_build.build(quiet=True)
    return flce.lib()


def test_exports_every_declared_symbol(L):
    names = flce.declared_functions()
    assert set(names) == {"flce_workspace_bytes", "flce_forward", "flce_backward",
                          "flce_read_status", "flce_status_string", "flce_instrument",
                          "flce_instrument_read", "flce_forward_noalloc", "flce_forward_fp8",
                          "flce_quantize_e4m3", "flce_selftest_wait_timeout",
                          "flce_count_valid", "flce_forward_dp", "flce_forward_dp_bucketed",
                          "flce_rmsnorm_forward",
                          "flce_rmsnorm_workspace_bytes", "flce_rmsnorm_backward",
                          "flce_workspace_bytes_rmsnorm", "flce_forward_rmsnorm",
                          "flce_scale_grads_rmsnorm", "flce_forward_rmsnorm_dp",
                          "flce_check_pair_schedule"}
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported


def test_library_is_built_for_sm100a():
    flags = flce_build.nvcc_flags()
    assert "arch=compute_100a,code=sm_100a" in flags


def test_status_strings(L):
    assert flce.status_string(0) == "FLCE_OK"
    for code in (-1, -2, -3, -4, -5, -6):
        assert flce.status_string(code).startswith("FLCE_ERR")


def test_workspace_has_no_tokens_by_vocab_term(L):
    s = flce.make_shape(65536, 3072, 50304, 50257, 15.0, -1, 0)
    fwd = flce.workspace_bytes(s, False)
    grads = flce.workspace_bytes(s, True)
    logits_bytes = 65536 * 50304 * 2                     # one bf16 N x Vpad buffer
    W_bytes = 50304 * 3072 * 2
    assert 0 < fwd < grads < logits_bytes / 6
    assert grads < 3 * W_bytes                            # O(Vpad * chunk) with chunk <= 8192
    # doubling N grows the scratch only by O(N) per-row words, not by Vpad per row
    s2 = flce.make_shape(131072, 3072, 50304, 50257, 15.0, -1, 0)
    assert flce.workspace_bytes(s2, True) - grads < 32 * 65536
    # the chunk bounds the gradient operand
    s3 = flce.make_shape(65536, 3072, 50304, 50257, 15.0, -1, 1024)
    assert flce.workspace_bytes(s3, True) < grads / 3


def test_invalid_shapes_give_zero_workspace(L):
    for bad in [dict(N=-1), dict(d=0), dict(Vreal=60000), dict(Vreal=0), dict(chunk_rows=-4)]:
        kw = dict(N=8, d=64, Vpad=128, Vreal=100, cap=15.0, ignore_index=-1, chunk_rows=0)
        kw.update(bad)
        s = flce.make_shape(**kw)
        assert flce.workspace_bytes(s, True) == 0, bad


def test_host_rejects_bad_arguments_before_launch(L):
    """These return before any CUDA call, so they run without a GPU."""
    s = flce.make_shape(8, 64, 128, 100)
    ws = flce.workspace_bytes(s, True)
    good = 0x10000000  # never dereferenced: every call below fails validation first
    args = dict(X=good, W=good, t=good, loss=good, lse=good, dX=good, dW=good, ws=good)

    def fwd(**over):
        a = dict(args)
        a.update(over)
        return flce.raw_forward(s, a["X"], a["W"], a["t"], a["loss"], a["lse"], 1,
                                over.get("g"), a["dX"], a["dW"], over.get("dtype", 0), 0,
                                a["ws"], over.get("ws_bytes", ws), None)

    assert fwd(X=None) == -1
    assert fwd(t=None) == -1
    assert fwd(loss=None) == -1
    assert fwd(dW=None) == -1
    assert fwd(X=good + 2) == -2
    assert fwd(ws=good + 16) == -2                 # workspace must be 256-byte aligned
    assert fwd(ws_bytes=ws - 1) == -3
    assert fwd(dtype=2) == -1                      # dW element type other than fp32 / bf16
    assert fwd(g=good + 2) == -2                   # grad_scale not 4-byte aligned
    bad_d = flce.make_shape(8, 60, 128, 100)
    assert flce.raw_forward(bad_d, good, good, good, good, good, 0, None, None, None, 0, 0, good,
                            1 << 30, None) == -2
    assert flce.raw_backward(s, good, good, good, None, None, good, good, 0, 0, 0, good, ws,
                             None) == -1       # lse missing on the recompute path
    assert flce.raw_backward(s, good, good, good, good, None, None, good, 0, 0, 0, good, ws,
                             None) == -1
    assert flce.raw_backward(s, good, good, good, good, None, good, good, 3, 0, 0, good, ws,
                             None) == -1       # bad dW element type
    # an accumulated dW cannot be scaled after the fact: g belongs in the forward's grad_scale
    assert flce.raw_backward(s, good, good, good, good, good, good, good, 0, 1, 1, None, 0,
                             None) == -1


def test_instrumentation_counters_without_gpu(L):
    flce.instrument(True)
    st = flce.instrument_read()
    flce.instrument(False)
    assert st["launches_total"] == 0
    assert all(v["launches"] == 0 and v["ms"] == 0 for v in st["gemm"].values())


def test_selftest_rejects_bad_limits(L):
    p = 0x10000000      # never dereferenced: argument checks come first
    assert L.flce_selftest_wait_timeout(None, 1000, None) == -1
    assert L.flce_selftest_wait_timeout(p, 0, None) == -1
    assert L.flce_selftest_wait_timeout(p, 11_000_000_000, None) == -1
    assert L.flce_selftest_wait_timeout(p + 16, 1000, None) == -2


def test_shape_struct_matches_header():
    # int64 N, d, Vpad, Vreal; float cap (+4 padding); int64 ignore_index, chunk_rows
    assert ctypes.sizeof(_abi.flce_shape) == 56
    assert _abi.flce_shape.cap.offset == 32 and _abi.flce_shape.ignore_index.offset == 40


def test_rmsnorm_and_quantiser_reject_bad_arguments_before_launch(L):
    p = 0x10000000      # never dereferenced: argument checks come first
    fwd = L.flce_rmsnorm_forward
    fwd.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_int64,
                    ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert fwd(p, None, 1e-6, 4, 64, p, p, None) == -1          # gamma missing
    assert fwd(p, p, -1.0, 4, 64, p, p, None) == -1             # negative eps
    assert fwd(p, p, 1e-6, 4, 60, p, p, None) == -2             # d % 8 != 0
    assert fwd(p + 8, p, 1e-6, 4, 64, p, p, None) == -2         # H not 16-byte aligned
    assert fwd(p, p, 1e-6, 4, 64, p, p + 2, None) == -2         # rstd not 4-byte aligned
    bwd = L.flce_rmsnorm_backward
    ws = flce.lib().flce_rmsnorm_workspace_bytes(300, 64)
    assert ws >= 3 * 64 * 4
    assert bwd(p, p, p, p, 300, 64, p, p, 0, p, ws - 1, None) == -3
    assert bwd(p, p, p + 2, p, 300, 64, p, p, 0, p, ws, None) == -2
    assert bwd(p, p, p, p, 300, 64, p, None, 0, p, ws, None) == -1
    q = L.flce_quantize_e4m3
    assert q(p, -1, p, p, None) == -1
    assert q(p, 16, None, p, None) == -1
    assert q(p, 16, p, p + 2, None) == -2


def test_rmsnorm_head_rejects_bad_arguments_before_launch(L):
    p = 0x10000000      # never dereferenced: argument checks come first
    s = flce.make_shape(8, 64, 128, 100)
    sp = ctypes.byref(s)
    ws = L.flce_workspace_bytes_rmsnorm(sp, 1)
    # beyond the head's workspace: the normalised rows and rstd, and the fold's partials
    assert ws >= flce.workspace_bytes(s, True) + 8 * 64 * 2 + 8 * 4
    f = L.flce_forward_rmsnorm
    # H, gamma, eps, W, t, loss, lse, want_grads, g, dH, dgamma, dW, dW_dtype, acc, ws,
    # ws_bytes, stream
    assert f(sp, p, None, 1e-6, p, p, p, p, 1, None, p, p, p, 0, 0, p, ws, None) == -1  # gamma
    assert f(sp, p, p, -1.0, p, p, p, p, 1, None, p, p, p, 0, 0, p, ws, None) == -1     # eps
    assert f(sp, None, p, 1e-6, p, p, p, p, 1, None, p, p, p, 0, 0, p, ws, None) == -1  # H
    assert f(sp, p + 8, p, 1e-6, p, p, p, p, 1, None, p, p, p, 0, 0, p, ws, None) == -2
    assert f(sp, p, p, 1e-6, p, p, p, p, 1, None, p, p, p, 0, 0, p, ws - 1, None) == -3
    assert f(sp, p, p, 1e-6, p, p, p, p, 1, None, p, None, p, 0, 0, p, ws, None) == -1  # dgamma
    assert f(sp, p, p, 1e-6, p, p, p, p, 1, None, p, p + 2, p, 0, 0, p, ws, None) == -2
    assert f(sp, p, p, 1e-6, p, p, p, p, 1, None, p, p, p, 5, 0, p, ws, None) == -1    # dtype
    fd = L.flce_forward_rmsnorm_dp
    # H, gamma, eps, W, t, n_valid_total, loss, lse, want_grads, g, dH, dgamma, dW, dtype, acc,
    # ws, ws_bytes, stream
    assert fd(sp, p, p, 1e-6, p, p, None, p, p, 1, None, p, p, p, 0, 0, p, ws, None) == -1
    assert fd(sp, p, p, 1e-6, p, p, p + 4, p, p, 1, None, p, p, p, 0, 0, p, ws, None) == -2
    assert fd(sp, p, p, 1e-6, p, p, p, p, p, 1, None, p, None, p, 0, 0, p, ws, None) == -1
    sg = L.flce_scale_grads_rmsnorm
    assert sg(sp, p, p, None, p, 0, None) == -1
    assert sg(sp, p, p, p, p, 2, None) == -1
    assert sg(sp, p + 2, p, p, p, 0, None) == -2
    assert sg(sp, p, p + 8, p, p, 0, None) == -2


def test_fp8_dp_and_count_entry_points_reject_bad_arguments_before_launch(L):
    p = 0x10000000      # never dereferenced: argument checks come first
    s = flce.make_shape(8, 64, 128, 100)
    ws = flce.workspace_bytes(s, True)
    sp = ctypes.byref(s)
    f8 = L.flce_forward_fp8
    # X8, W8, sx, sw, X, W, t, loss, lse, want_grads, grad_fp8, g, dX, dW, dW_dtype, acc, ws,
    # ws_bytes, stream
    assert f8(sp, p, p, None, p, p, p, p, p, p, 1, 0, None, p, p, 0, 0, p, ws, None) == -1  # sx
    assert f8(sp, p, p, p, p, None, p, p, p, p, 1, 0, None, p, p, 0, 0, p, ws, None) == -1  # X
    assert f8(sp, p, p, p + 2, p, p, p, p, p, p, 1, 0, None, p, p, 0, 0, p, ws, None) == -2
    assert f8(sp, p + 8, p, p, p, p, p, p, p, p, 1, 0, None, p, p, 0, 0, p, ws, None) == -2
    assert f8(sp, p, p, p, p, p, p, p, p, p, 1, 0, None, p, p, 0, 0, p, ws - 1, None) == -3
    # 8-bit gradients need the cap as exp reference: no softcap (cap 0) or cap > 32 is refused
    for cap in (0.0, 40.0):
        sc = flce.make_shape(8, 64, 128, 100, cap)
        assert f8(ctypes.byref(sc), p, p, p, p, None, None, p, p, p, 1, 1, None, p, p, 0, 0, p,
                  flce.workspace_bytes(sc, True), None) == -1
    s48 = flce.make_shape(8, 72, 128, 100)          # d % 16 != 0: e4m3 rows not 16-byte
    assert f8(ctypes.byref(s48), p, p, p, p, p, p, p, p, p, 0, 0, None, None, None, 0, 0, p,
              1 << 30, None) == -2
    dp = L.flce_forward_dp
    # X, W, t, nv_total, loss, lse, want_grads, g, dX, dW, dW_dtype, acc, ws, ws_bytes, stream
    assert dp(sp, p, p, p, None, p, p, 1, None, p, p, 0, 0, p, ws, None) == -1    # count
    assert dp(sp, p, p, p, p + 4, p, p, 1, None, p, p, 0, 0, p, ws, None) == -2   # 8-byte
    cv = L.flce_count_valid
    assert cv(sp, p, None, None) == -1
    assert cv(sp, p, p + 4, None) == -2
    bad = flce.make_shape(8, 64, 128, 200)          # Vreal > Vpad
    assert cv(ctypes.byref(bad), p, p, None) == -1


def test_bucketed_entry_point_rejects_bad_arguments_before_launch(L):
    p = 0x10000000      # never dereferenced: argument checks come first
    s = flce.make_shape(8, 64, 1024, 1000)          # 4 vocabulary tiles of 256 rows
    ws = flce.workspace_bytes(s, True)
    f = L.flce_forward_dp_bucketed
    P = ctypes.c_void_p

    def call(n, events, bounds=True, nv=p):
        ev = (P * max(n, 1))(*([p] * max(n, 1))) if events else None
        bd = (ctypes.c_int64 * (max(n, 1) + 1))() if bounds else None
        return f(ctypes.byref(s), p, p, p, nv, p, p, None, p, p, 0, 0, n, ev, bd, p, ws, None)

    assert call(0, True) == -1                       # at least one bucket
    assert call(5, True) == -1                       # more buckets than vocabulary tiles
    assert call(2, False) == -1                      # events missing
    assert call(2, True, bounds=False) == -1         # bounds missing
    assert call(2, True, nv=None) == -1              # global count missing
    assert call(2, True, nv=p + 4) == -2             # count not 8-byte aligned
    null_event = (P * 2)(p, None)
    bd = (ctypes.c_int64 * 3)()
    assert f(ctypes.byref(s), p, p, p, p, p, p, None, p, p, 0, 0, 2, null_event, bd, p, ws,
             None) == -1
