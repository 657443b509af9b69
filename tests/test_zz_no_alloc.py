"""flce_forward_noalloc: the statistics-only forward (loss and per-row lse) whose scratch is a
fixed device array inside the library, for callers that cannot allocate device memory at call
time (a plugin whose host framework owns all device memory and gives it no allocator, or a
caller that must not risk the device synchronisation cudaMalloc may cause).

Its outputs are checked against the fp64 oracle (and against flce_forward, which uses a caller
workspace) within the tolerances of the other parity tests, on calls in a row (the array keeps
the previous call's contents), on a shape that runs several chunks through the array, and on
one so large that the automatic chunk drops below 4096 rows.  The device status word is read
back with flce_read_status(NULL, ...).  This file is collected last so that a run stopping at
the first failure has already run every other test."""
import numpy as np
import pytest

import oracle
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


def _call(X, W, t, c, chunk_rows=0):
    """flce_forward_noalloc through the C ABI; returns (loss, lse [N] float64, status, n_valid)."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    N = X.shape[0]
    loss = torch.full((), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    shape = flce.make_shape(N, c.d, c.Vpad, c.Vreal, c.cap, c.ignore_index, chunk_rows)
    rc = flce.raw_forward_noalloc(shape, X.data_ptr(), W.data_ptr(), t.data_ptr(),
                                  loss.data_ptr(), lse.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    assert rc == 0, flce.status_string(rc)
    status, nv = flce.read_status(None)           # the fixed scratch's header; synchronises
    return float(loss.item()), lse.double().cpu().numpy(), status, nv


def _noalloc(inp, chunk_rows=0):
    c = inp["cfg"]
    return _call(_dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"]), c, chunk_rows)


def _oracle(inp):
    c = inp["cfg"]
    return oracle.forward(synth.bf16_to_f64(inp["X"]), synth.bf16_to_f64(inp["W"]),
                          inp["targets"], c.Vreal, c.cap, c.ignore_index)


def _with_workspace(inp):
    import torch
    import lm_head_linear_gemm_b200 as flce
    c = inp["cfg"]
    loss, lse, _, _, _ = flce.forward(_dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"]),
                                      c.Vreal, c.cap, c.ignore_index, False)
    torch.cuda.synchronize()
    return float(loss.item()), lse.double().cpu().numpy()


def _check(got, ref):
    loss, lse, status, nv = got
    assert status == 0 and nv == ref["n_valid"]
    assert abs(loss - ref["loss"]) <= LOSS_TOL, (loss, ref["loss"])
    assert np.all(np.isfinite(lse))
    assert np.abs(lse - ref["lse"]).max() <= LSE_TOL


def test_noalloc_matches_oracle_on_calls_in_a_row(cuda_device):
    first = synth.make_inputs("small", N=3000)          # the pages' vocabulary, d = 1536
    second = synth.make_inputs(synth.custom_config("ragged", N=300, d=200, Vreal=1500,
                                                   Vpad=1544, w_std=0.05, ignore_count=7))
    for inp in (first, second, first):
        got = _noalloc(inp)
        _check(got, _oracle(inp))
        ref_loss, ref_lse = _with_workspace(inp)
        assert abs(got[0] - ref_loss) <= LOSS_TOL
        assert np.abs(got[1] - ref_lse).max() <= LSE_TOL


def test_noalloc_several_chunks_through_the_array(cuda_device):
    """1000 rows in chunks of 128 (the last one ragged): eight passes reuse the array."""
    inp = synth.make_inputs(synth.custom_config("chunks", N=1000, d=256, Vreal=3000, Vpad=3008,
                                                w_std=0.05, ignore_count=11))
    _check(_noalloc(inp, chunk_rows=128), _oracle(inp))


def test_noalloc_automatic_chunk_below_4096_rows(cuda_device):
    """200,704 rows at the 3.8b head's shape (d = 3072, Vpad = 50304): the per-row scratch no
    longer leaves room for 4096-row chunks, so the call picks 2048.  The rows are 392 copies of a
    512-row base problem, so the oracle on the base fixes every result: the loss and each row's
    lse equal the base's, and copies of a row agree bit for bit.  One base target is out of
    range: the status word must carry the bad-target bit and every copy counts it as ignored."""
    import torch
    k, base = 392, 512
    inp = synth.make_inputs("3.8b", N=base)
    t = inp["targets"].copy()
    t[5] = 60000                                   # not a vocabulary id
    inp = dict(inp, targets=t)
    c = inp["cfg"]
    ref = _oracle(inp)
    assert ref["n_bad"] == 1
    X = _dev(inp["X"]).repeat(k, 1)
    tt = _dev(t).repeat(k)
    W = _dev(inp["W"])
    loss, lse, status, nv = _call(X, W, tt, c)
    assert status & 1
    assert nv == k * ref["n_valid"]
    assert abs(loss - ref["loss"]) <= LOSS_TOL
    lse_k = lse.reshape(k, base)
    assert np.array_equal(lse_k, np.broadcast_to(lse_k[:1], lse_k.shape))
    assert np.abs(lse_k[0] - ref["lse"]).max() <= LSE_TOL
    del X
    torch.cuda.empty_cache()


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    import lm_head_linear_gemm_b200 as flce
    # 16384 rows at d = 3072 fit; ten million rows need ~200 MB of per-row scratch and do not.
    big = flce.make_shape(10_000_000, 3072, 50304, 50257, 15.0, -1, 0)
    p = 0x10000000   # never dereferenced: the size check fails before anything runs
    assert flce.raw_forward_noalloc(big, p, p, p, p, p, None) == -3
    wide_chunk = flce.make_shape(16384, 3072, 50304, 50257, 15.0, -1, 8192)
    assert flce.raw_forward_noalloc(wide_chunk, p, p, p, p, p, None) == -3
