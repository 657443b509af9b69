"""flce_forward_noalloc: the statistics-only forward (loss and per-row lse) whose scratch is a
fixed device array inside the library, for callers that cannot allocate device memory at call
time (a plugin whose host framework owns all device memory and gives it no allocator, or a
caller that must not risk the device synchronisation cudaMalloc may cause).

Its outputs must match flce_forward (want_grads = 0), which uses a caller workspace, within the
tolerances of the other parity tests, on two calls in a row (the array keeps the previous call's
contents).  This file is collected last so that a run stopping at the first failure has already
run every other test."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

LOSS_TOL = 2e-3
LSE_TOL = 2e-3


def _dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _noalloc(inp):
    import torch
    import lm_head_linear_gemm_b200 as flce
    c = inp["cfg"]
    X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"])
    loss = torch.full((), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((c.N,), float("nan"), dtype=torch.float32, device="cuda")
    shape = flce.make_shape(c.N, c.d, c.Vpad, c.Vreal, c.cap, c.ignore_index, 0)
    rc = flce.raw_forward_noalloc(shape, X.data_ptr(), W.data_ptr(), t.data_ptr(),
                                  loss.data_ptr(), lse.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    assert rc == 0, flce.status_string(rc)
    torch.cuda.synchronize()
    return float(loss.item()), lse.double().cpu().numpy()


def _with_workspace(inp):
    import torch
    import lm_head_linear_gemm_b200 as flce
    c = inp["cfg"]
    loss, lse, _, _, _ = flce.forward(_dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"]),
                                      c.Vreal, c.cap, c.ignore_index, False)
    torch.cuda.synchronize()
    return float(loss.item()), lse.double().cpu().numpy()


def test_noalloc_matches_workspace_forward_twice(cuda_device):
    first = synth.make_inputs("small", N=3000)          # the pages' vocabulary, d = 1536
    second = synth.make_inputs(synth.custom_config("ragged", N=300, d=200, Vreal=1500,
                                                   Vpad=1544, w_std=0.05, ignore_count=7))
    for inp in (first, second):
        got_loss, got_lse = _noalloc(inp)
        ref_loss, ref_lse = _with_workspace(inp)
        assert abs(got_loss - ref_loss) <= LOSS_TOL
        assert np.all(np.isfinite(got_lse))
        assert np.abs(got_lse - ref_lse).max() <= LSE_TOL


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    import lm_head_linear_gemm_b200 as flce
    # 16384 rows at d = 3072 fit; ten million rows need ~200 MB of per-row scratch and do not.
    big = flce.make_shape(10_000_000, 3072, 50304, 50257, 15.0, -1, 0)
    p = 0x10000000   # never dereferenced: the size check fails before anything runs
    assert flce.raw_forward_noalloc(big, p, p, p, p, p, None) == -3
    wide_chunk = flce.make_shape(16384, 3072, 50304, 50257, 15.0, -1, 8192)
    assert flce.raw_forward_noalloc(wide_chunk, p, p, p, p, p, None) == -3
