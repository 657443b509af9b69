"""flce_forward_dp on the GPU against the fp64 oracle on the union batch.

Ranks are emulated in one process with no collective: each rank's call is normalised by the
count of rows in the loss over all ranks, so its loss share, its dX rows and its dW
contribution must add up to the oracle's loss, dX and dW of the union of all ranks' rows --
also when one rank has no row in the loss (its own count is 0, the global one is not).  dp_step
runs through a world-size-1 NCCL process group and is compared with the oracle as well."""
import os
import socket

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

LOSS_TOL = 2e-3
LSE_TOL = 2e-3
REL_L2 = 1e-2


def _dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _oracle(inp, t):
    c = inp["cfg"]
    return oracle.forward_backward(synth.bf16_to_f64(inp["X"]), synth.bf16_to_f64(inp["W"]), t,
                                   c.Vreal, c.cap, -1)


@pytest.mark.parametrize("parts,ignored_part", [([(0, 300), (300, 1000)], None),
                                                ([(0, 256), (256, 600), (600, 1000)], None),
                                                ([(0, 300), (300, 1000)], 0)])
def test_rank_shares_match_the_oracle_on_the_union_batch(cuda_device, parts, ignored_part):
    import torch
    import lm_head_linear_gemm_b200 as flce
    from lm_head_linear_gemm_b200.data_parallel import LibraryOps
    inp = synth.make_inputs("small", N=1000)
    c = inp["cfg"]
    t_np = inp["targets"].copy()
    if ignored_part is not None:
        a, b = parts[ignored_part]
        t_np[a:b] = -1                       # this rank's own count is 0
    ref = _oracle(inp, t_np)
    X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(t_np)
    ops = LibraryOps()
    nv = sum(ops.count_valid(t[a:b].contiguous(), c.Vreal, -1) for a, b in parts)
    shares, dXs, lses, dWsum = [], [], [], torch.zeros(W.shape, device="cuda")
    for a, b in parts:
        l, lse, dXp, dWp, _ = flce.forward_dp(X[a:b].contiguous(), W, t[a:b].contiguous(), nv,
                                              c.Vreal, c.cap, -1, True, chunk_rows=256)
        shares.append(float(l.item()))
        dXs.append(dXp.double().cpu().numpy())
        lses.append(lse.double().cpu().numpy())
        dWsum += dWp
    torch.cuda.synchronize()
    assert int(nv.item()) == ref["n_valid"]
    assert abs(sum(shares) - ref["loss"]) <= LOSS_TOL
    if ignored_part is not None:
        assert shares[ignored_part] == 0.0
        assert np.abs(dXs[ignored_part]).max() == 0.0
    assert np.abs(np.concatenate(lses) - ref["lse"]).max() <= LSE_TOL
    assert _rel(np.concatenate(dXs), ref["dX"]) <= REL_L2
    assert _rel(dWsum.double().cpu().numpy(), ref["dW"]) <= REL_L2


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
        ref = _oracle(inp, inp["targets"])
        X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"])
        loss, lse, dX, dW, nv = flce.dp_step(X, W, t, c.Vreal, c.cap, -1)
        torch.cuda.synchronize()
        assert int(nv.item()) == ref["n_valid"] == 293
        assert abs(loss.item() - ref["loss"]) <= LOSS_TOL
        assert np.abs(lse.double().cpu().numpy() - ref["lse"]).max() <= LSE_TOL
        assert _rel(dX.double().cpu().numpy(), ref["dX"]) <= REL_L2
        assert _rel(dW.double().cpu().numpy(), ref["dW"]) <= REL_L2
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_buckets,chunk_rows", [(4, 0), (3, 256), (7, 128)])
def test_bucketed_forward_matches_oracle_and_unbucketed(cuda_device, n_buckets, chunk_rows):
    """flce_forward_dp_bucketed: the last chunk's dW in vocabulary buckets, each marked by an
    event.  The buckets tile [0, Vpad) in whole 256-row vocabulary tiles, every event has fired
    once the stream is done, and the results equal the unbucketed call bit for bit (the same
    tiles in the same order, only spread over more launches) and the oracle within tolerance."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    from lm_head_linear_gemm_b200.data_parallel import LibraryOps
    inp = synth.make_inputs("small", N=700)
    c = inp["cfg"]
    ref = _oracle(inp, inp["targets"])
    X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"])
    nv = LibraryOps().count_valid(t, c.Vreal, -1)
    events = [torch.cuda.Event() for _ in range(n_buckets)]
    loss, lse, dX, dW, bounds, _ = flce.forward_dp_bucketed(X, W, t, nv, c.Vreal, c.cap, -1,
                                                            events, chunk_rows=chunk_rows)
    l2, lse2, dX2, dW2, _ = flce.forward_dp(X, W, t, nv, c.Vreal, c.cap, -1, True,
                                            chunk_rows=chunk_rows)
    torch.cuda.synchronize()
    assert bounds[0] == 0 and bounds[-1] == c.Vpad and len(bounds) == n_buckets + 1
    assert all(b % 256 == 0 for b in bounds[:-1]) and all(np.diff(bounds) > 0)
    assert all(ev.query() for ev in events)
    assert torch.equal(loss, l2) and torch.equal(lse, lse2)
    assert torch.equal(dX, dX2) and torch.equal(dW, dW2)
    assert abs(loss.item() - ref["loss"]) <= LOSS_TOL
    assert _rel(dX.double().cpu().numpy(), ref["dX"]) <= REL_L2
    assert _rel(dW.double().cpu().numpy(), ref["dW"]) <= REL_L2


def test_bucketed_forward_bf16_dW_accumulated(cuda_device):
    """The bucketed launches writing a bf16 dW (the bucket offsets are in 2-byte elements) and
    adding into it: equal bit for bit to the unbucketed call, and the sum of the two calls'
    gradients (grad_scale 1/2 each) matches the oracle."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    from lm_head_linear_gemm_b200.data_parallel import LibraryOps
    inp = synth.make_inputs("small", N=700)
    c = inp["cfg"]
    ref = _oracle(inp, inp["targets"])
    X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"])
    nv = LibraryOps().count_valid(t, c.Vreal, -1)
    events = [torch.cuda.Event() for _ in range(5)]
    dWb = torch.zeros(W.shape, dtype=torch.bfloat16, device="cuda")
    dWu = torch.zeros(W.shape, dtype=torch.bfloat16, device="cuda")
    for k in range(2):
        flce.forward_dp_bucketed(X, W, t, nv, c.Vreal, c.cap, -1, events, dW=dWb,
                                 accumulate_dW=k > 0, chunk_rows=256, grad_scale=0.5)
        flce.forward_dp(X, W, t, nv, c.Vreal, c.cap, -1, True, dW=dWu, accumulate_dW=k > 0,
                        chunk_rows=256, grad_scale=0.5)
    torch.cuda.synchronize()
    assert torch.equal(dWb, dWu)
    assert _rel(dWb.double().cpu().numpy(), ref["dW"]) <= REL_L2


def test_dp_step_bucketed_world_size_one_nccl(cuda_device):
    """dp_step with the dW all-reduce in four buckets on a communication stream (NCCL, world
    size 1) against the oracle."""
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
        inp = synth.make_inputs("small", N=600)
        c = inp["cfg"]
        ref = _oracle(inp, inp["targets"])
        X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"])
        loss, lse, dX, dW, nv = flce.dp_step(X, W, t, c.Vreal, c.cap, -1, buckets=4,
                                             chunk_rows=256)
        torch.cuda.synchronize()
        assert int(nv.item()) == ref["n_valid"]
        assert abs(loss.item() - ref["loss"]) <= LOSS_TOL
        assert _rel(dX.double().cpu().numpy(), ref["dX"]) <= REL_L2
        assert _rel(dW.double().cpu().numpy(), ref["dW"]) <= REL_L2
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("parts,ignored_part", [([(0, 300), (300, 1000)], None),
                                                ([(0, 300), (300, 1000)], 1)])
def test_rmsnorm_rank_shares_match_the_oracle_on_the_union_batch(cuda_device, parts,
                                                                  ignored_part):
    """flce_forward_rmsnorm_dp: each emulated rank's loss share, its dH rows and its dgamma and
    dW contributions add up to one oracle step of the final RMSNorm and the head on the union
    of the ranks' rows (also when one rank has no row in the loss)."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    from lm_head_linear_gemm_b200.data_parallel import LibraryOps
    inp = synth.make_rmsnorm_inputs("small", N=1000)
    c = inp["cfg"]
    t_np = inp["targets"].copy()
    if ignored_part is not None:
        a, b = parts[ignored_part]
        t_np[a:b] = -1
    ref = oracle.rmsnorm_head(synth.bf16_to_f64(inp["H"]), synth.bf16_to_f64(inp["gamma"]),
                              synth.bf16_to_f64(inp["W"]), t_np, c.Vreal, c.cap, -1)
    H, gamma, W, t = _dev(inp["H"]), _dev(inp["gamma"]), _dev(inp["W"]), _dev(t_np)
    ops = LibraryOps()
    nv = sum(ops.count_valid(t[a:b].contiguous(), c.Vreal, -1) for a, b in parts)
    shares, dHs, lses = [], [], []
    dgsum = torch.zeros(c.d, device="cuda")
    dWsum = torch.zeros(W.shape, device="cuda")
    for a, b in parts:
        l, lse, dH, dg, dW, _ = flce.forward_rmsnorm(H[a:b].contiguous(), gamma, W,
                                                     t[a:b].contiguous(), c.Vreal, c.cap, -1,
                                                     1e-6, True, chunk_rows=256,
                                                     n_valid_total=nv)
        shares.append(float(l.item()))
        dHs.append(dH.double().cpu().numpy())
        lses.append(lse.double().cpu().numpy())
        dgsum += dg
        dWsum += dW
    torch.cuda.synchronize()
    assert int(nv.item()) == ref["n_valid"]
    assert abs(sum(shares) - ref["loss"]) <= LOSS_TOL
    if ignored_part is not None:
        assert shares[ignored_part] == 0.0
        assert np.abs(dHs[ignored_part]).max() == 0.0
    assert np.abs(np.concatenate(lses) - ref["lse"]).max() <= LSE_TOL
    assert _rel(np.concatenate(dHs), ref["dH"]) <= REL_L2
    assert _rel(dgsum.double().cpu().numpy(), ref["dgamma"]) <= REL_L2
    assert _rel(dWsum.double().cpu().numpy(), ref["dW"]) <= REL_L2


def test_dp_step_rmsnorm_world_size_one_nccl(cuda_device):
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
        inp = synth.make_rmsnorm_inputs(synth.custom_config("ragged", N=300, d=200, Vreal=1500,
                                                            Vpad=1544, w_std=0.05,
                                                            ignore_count=7))
        c = inp["cfg"]
        ref = oracle.rmsnorm_head(synth.bf16_to_f64(inp["H"]), synth.bf16_to_f64(inp["gamma"]),
                                  synth.bf16_to_f64(inp["W"]), inp["targets"], c.Vreal, c.cap,
                                  -1)
        loss, lse, dH, dg, dW, nv = flce.dp_step_rmsnorm(_dev(inp["H"]), _dev(inp["gamma"]),
                                                         _dev(inp["W"]), _dev(inp["targets"]),
                                                         c.Vreal, c.cap, -1)
        torch.cuda.synchronize()
        assert int(nv.item()) == ref["n_valid"] == 293
        assert abs(loss.item() - ref["loss"]) <= LOSS_TOL
        assert np.abs(lse.double().cpu().numpy() - ref["lse"]).max() <= LSE_TOL
        assert _rel(dH.double().cpu().numpy(), ref["dH"]) <= REL_L2
        assert _rel(dg.double().cpu().numpy(), ref["dgamma"]) <= REL_L2
        assert _rel(dW.double().cpu().numpy(), ref["dW"]) <= REL_L2
    finally:
        dist.destroy_process_group()
