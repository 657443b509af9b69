"""flce_forward_dp on the GPU: per-rank calls normalised by the global count add up to one call
on the union batch (emulated ranks in one process, no collective), and dp_step runs through a
world-size-1 NCCL process group."""
import os
import socket

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def test_rank_shares_add_up_to_the_union_batch(cuda_device):
    import torch
    import lm_head_linear_gemm_b200 as flce
    from lm_head_linear_gemm_b200.data_parallel import LibraryOps
    inp = synth.make_inputs("small", N=1000)
    c = inp["cfg"]
    X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"])
    loss, lse, dX, dW, _ = flce.forward(X, W, t, c.Vreal, c.cap, -1, True)
    ops = LibraryOps()
    parts = [(0, 300), (300, 1000)]
    nv = sum(ops.count_valid(t[a:b], c.Vreal, -1) for a, b in parts)
    shares, dXs, dWsum = [], [], torch.zeros_like(dW)
    for a, b in parts:
        l, _, dXp, dWp, _ = flce.forward_dp(X[a:b].contiguous(), W, t[a:b].contiguous(), nv,
                                            c.Vreal, c.cap, -1, True)
        shares.append(l)
        dXs.append(dXp)
        dWsum += dWp
    torch.cuda.synchronize()
    assert int(nv.item()) == int((inp["targets"] != -1).sum())
    assert abs(float(sum(shares).item()) - float(loss.item())) < 1e-4
    assert _rel(torch.cat(dXs).double().cpu().numpy(), dX.double().cpu().numpy()) < 1e-3
    assert _rel(dWsum.double().cpu().numpy(), dW.double().cpu().numpy()) < 1e-5


def test_dp_step_world_size_one_nccl(cuda_device):
    import torch
    import torch.distributed as dist
    import lm_head_linear_gemm_b200 as flce
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        inp = synth.make_inputs(synth.custom_config("ragged", N=300, d=200, Vreal=1500,
                                                    Vpad=1544, w_std=0.05, ignore_count=7))
        c = inp["cfg"]
        X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"])
        loss, lse, dX, dW, nv = flce.dp_step(X, W, t, c.Vreal, c.cap, -1)
        ref_loss, _, ref_dX, ref_dW, _ = flce.forward(X, W, t, c.Vreal, c.cap, -1, True)
        torch.cuda.synchronize()
        assert int(nv.item()) == 293
        assert abs(loss.item() - ref_loss.item()) < 1e-6
        assert torch.equal(dX, ref_dX) and torch.equal(dW, ref_dW)
    finally:
        dist.destroy_process_group()
