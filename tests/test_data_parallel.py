"""The data-parallel exchange (dp_step) on world_size-2 gloo ranks on the CPU.

The device work is stood in for by the fp64 oracle (test-side only: ``OracleOps`` implements
the contract of flce_count_valid / flce_forward_dp); what is under test is the exchange:
counts all-reduced before the forward, loss shares and dW all-reduced after it.  The two-rank
result must equal a single oracle call on the union of both ranks' rows, also when the split
is uneven and when one rank has no row in the loss.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

VR, VP, D, CAP = 40, 48, 16, 15.0


class OracleOps:
    def count_valid(self, targets, Vreal, ignore_index):
        valid, _ = oracle.valid_rows(targets.numpy(), Vreal, ignore_index)
        return torch.tensor([int(valid.sum())], dtype=torch.int64)

    def forward(self, X, W, targets, n_valid_total, Vreal, cap, ignore_index, dW, accumulate_dW,
                workspace, chunk_rows):
        Xn, Wn, t = X.numpy(), W.numpy(), targets.numpy()
        nt = int(n_valid_total.item())
        f = oracle.forward(Xn, Wn, t, Vreal, cap, ignore_index)
        nl = f["n_valid"]
        g = nl / nt if nt else 0.0
        dX, dWl = oracle.backward(Xn, Wn, t, Vreal, cap, ignore_index, g=g, lse=f["lse"])
        loss = torch.tensor(f["loss"] * g, dtype=torch.float64)
        dWt = torch.from_numpy(dWl)
        if dW is not None and accumulate_dW:
            dWt = dW + dWt
        return loss, torch.from_numpy(f["lse"]), torch.from_numpy(dX), dWt, None


def _data(seed=0, N=30):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((N, D))
    W = rng.standard_normal((VP, D)) * 1.5
    t = rng.integers(0, VR, N)
    t[rng.permutation(N)[:4]] = -1
    return X, W, t


def _worker(rank, world, port, split, all_ignored_rank, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from lm_head_linear_gemm_b200.data_parallel import dp_step
        X, W, t = _data()
        t = t.copy()
        lo, hi = (0, split) if rank == 0 else (split, X.shape[0])
        if rank == all_ignored_rank:
            t[lo:hi] = -1
        Xr = torch.from_numpy(X[lo:hi].copy())
        tr = torch.from_numpy(t[lo:hi].copy())
        loss, lse, dX, dW, nv = dp_step(Xr, torch.from_numpy(W), tr, VR, CAP, -1, ops=OracleOps())
        q.put((rank, float(loss), dX.numpy(), dW.numpy(), int(nv.item()), t))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("split,all_ignored_rank", [(15, -1), (7, -1), (20, 1)])
def test_two_rank_exchange_equals_union_batch(split, all_ignored_rank):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, split, all_ignored_rank, q))
             for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X, W, t = _data()
    t = t.copy()
    if all_ignored_rank == 0:
        t[:split] = -1
    elif all_ignored_rank == 1:
        t[split:] = -1
    ref = oracle.forward_backward(X, W, t, VR, CAP, -1)
    for r in (0, 1):
        assert abs(res[r][1] - ref["loss"]) < 1e-12          # both ranks hold the global loss
        np.testing.assert_allclose(res[r][3], ref["dW"], atol=1e-14)
        assert res[r][4] == ref["n_valid"]
    dX = np.concatenate([res[0][2], res[1][2]])
    np.testing.assert_allclose(dX, ref["dX"], atol=1e-14)
