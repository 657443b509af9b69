"""Failure detection on the GPU without faulting it: the library's bounded pipeline wait is run
on a barrier nothing arrives at (a short limit); it must give up, report FLCE_DEV_TIMEOUT through
the status word, and leave the context usable for the next call.  Invalid targets are covered in
test_parity_gpu.py (status bit, rows ignored)."""
import time

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_device):
    import torch
    import lm_head_linear_gemm_b200 as flce
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    flce.selftest_wait_timeout(ws, 50_000_000)          # 50 ms
    status, _ = flce.read_status(ws)
    elapsed = time.time() - t0
    assert status & flce.DEV_TIMEOUT
    assert elapsed < 5.0
    # the context still works: a normal forward afterwards succeeds with a clean status
    inp = synth.make_inputs("tiny")
    c = inp["cfg"]
    dev = lambda a: (torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
                     if a.dtype == np.uint16 else torch.from_numpy(a)).cuda()
    loss, lse, dX, dW, ws2 = flce.forward(dev(inp["X"]), dev(inp["W"]), dev(inp["targets"]),
                                          c.Vreal, c.cap, c.ignore_index, True)
    torch.cuda.synchronize()
    status2, nv = flce.read_status(ws2)
    assert status2 == 0 and nv == 62 and np.isfinite(loss.item())
