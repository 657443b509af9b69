"""The data-parallel exchange (dp_step) on world_size-2 gloo ranks on the CPU.

The device work is stood in for by the fp64 oracle (test-side only: ``OracleOps`` implements
the contract of flce_count_valid / flce_forward_dp / flce_forward_dp_bucketed); what is under
test is the exchange: counts all-reduced before the forward, loss shares and dW all-reduced
after it, in one piece or in vocabulary buckets issued as asynchronous all-reduces.  The
two-rank result must equal a single oracle call on the union of both ranks' rows, also when the
split is uneven, when one rank has no row in the loss, and over two accumulated micro-batches
with the upstream gradient 1/2 passed to the forward.
"""
import os
import shutil
import tempfile

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
                workspace, chunk_rows, grad_scale=None):
        Xn, Wn, t = X.numpy(), W.numpy(), targets.numpy()
        nt = int(n_valid_total.item())
        f = oracle.forward(Xn, Wn, t, Vreal, cap, ignore_index)
        nl = f["n_valid"]
        share = nl / nt if nt else 0.0
        gs = 1.0 if grad_scale is None else float(grad_scale)
        dX, dWl = oracle.backward(Xn, Wn, t, Vreal, cap, ignore_index, g=share * gs,
                                  lse=f["lse"])
        loss = torch.tensor(f["loss"] * share, dtype=torch.float64)
        dWt = torch.from_numpy(dWl)
        if dW is not None and accumulate_dW:
            dWt = dW + dWt
        return loss, torch.from_numpy(f["lse"]), torch.from_numpy(dX), dWt, None

    def forward_buckets(self, X, W, targets, n_valid_total, Vreal, cap, ignore_index, dW,
                        accumulate_dW, workspace, chunk_rows, n_buckets, grad_scale=None):
        loss, lse, dX, dWt, _ = self.forward(X, W, targets, n_valid_total, Vreal, cap,
                                             ignore_index, dW, accumulate_dW, workspace,
                                             chunk_rows, grad_scale)
        edges = np.linspace(0, dWt.shape[0], n_buckets + 1).astype(int)
        return loss, lse, dX, dWt, [(slice(edges[b], edges[b + 1]), None)
                                    for b in range(n_buckets)]

    def forward_rmsnorm(self, H, gamma, W, targets, n_valid_total, Vreal, cap, ignore_index, eps,
                        dgamma, dW, accumulate, workspace, chunk_rows, grad_scale=None):
        t = targets.numpy()
        nt = int(n_valid_total.item())
        nl = int(oracle.valid_rows(t, Vreal, ignore_index)[0].sum())
        share = nl / nt if nt else 0.0
        gs = 1.0 if grad_scale is None else float(grad_scale)
        f = oracle.rmsnorm_head(H.numpy(), gamma.numpy(), W.numpy(), t, Vreal, cap, ignore_index,
                                eps, g=share * gs)
        dg, dWt = torch.from_numpy(f["dgamma"]), torch.from_numpy(f["dW"])
        if accumulate:
            dg, dWt = dgamma + dg, dW + dWt
        return (torch.tensor(f["loss"] * share, dtype=torch.float64), torch.from_numpy(f["lse"]),
                torch.from_numpy(f["dH"]), dg, dWt)

    def allreduce_async(self, t, ready, group):
        return dist.all_reduce(t, group=group, async_op=True)


def _data(seed=0, N=30):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((N, D))
    W = rng.standard_normal((VP, D)) * 1.5
    t = rng.integers(0, VR, N)
    t[rng.permutation(N)[:4]] = -1
    return X, W, t


def _worker(rank, world, store_path, split, all_ignored_rank, buckets, micro, q):
    # a file rendezvous: no port that another process could take between its choice and use
    dist.init_process_group("gloo", init_method=f"file://{store_path}", rank=rank,
                            world_size=world)
    try:
        from lm_head_linear_gemm_b200.data_parallel import dp_step
        X, W, t = _data()
        t = t.copy()
        lo, hi = (0, split) if rank == 0 else (split, X.shape[0])
        if rank == all_ignored_rank:
            t[lo:hi] = -1
        Xr = torch.from_numpy(X[lo:hi].copy())
        tr = torch.from_numpy(t[lo:hi].copy())
        Wt = torch.from_numpy(W)
        if micro == 1:
            loss, lse, dX, dW, nv = dp_step(Xr, Wt, tr, VR, CAP, -1, ops=OracleOps(),
                                            buckets=buckets)
        else:
            # the same rows as `micro` micro-batches (halves of this rank's rows), dW
            # accumulated with grad_scale 1/micro and all-reduced after the last one
            cut = [lo + (hi - lo) * k // micro for k in range(micro + 1)]
            dW, dXs, losses = None, [], []
            for k in range(micro):
                a, b = cut[k] - lo, cut[k + 1] - lo
                loss, lse, dXk, dW, nv = dp_step(Xr[a:b], Wt, tr[a:b], VR, CAP, -1,
                                                 ops=OracleOps(), dW=dW, accumulate_dW=k > 0,
                                                 allreduce_dW=k == micro - 1,
                                                 grad_scale=1.0 / micro, buckets=buckets)
                dXs.append(dXk)
                losses.append(float(loss))
            dX = torch.cat(dXs)
            loss = losses
        q.put((rank, loss, dX.numpy(), dW.numpy(), int(nv.item()), t))
    finally:
        dist.destroy_process_group()


def _run(split, all_ignored_rank, buckets, micro):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    store_dir = tempfile.mkdtemp(prefix="flce_gloo_")
    store_path = os.path.join(store_dir, "rendezvous")
    procs = [ctx.Process(target=_worker,
                         args=(r, 2, store_path, split, all_ignored_rank, buckets, micro, q))
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
    shutil.rmtree(store_dir, ignore_errors=True)
    return res


@pytest.mark.parametrize("split,all_ignored_rank,buckets", [(15, -1, 1), (7, -1, 1),
                                                            (20, 1, 1), (15, -1, 4),
                                                            (20, 1, 3)])
def test_two_rank_exchange_equals_union_batch(split, all_ignored_rank, buckets):
    res = _run(split, all_ignored_rank, buckets, 1)
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


@pytest.mark.parametrize("buckets", [1, 4])
def test_two_rank_accumulation_over_micro_batches(buckets):
    """Each rank's rows as two micro-batches with grad_scale 1/2 and dW accumulated; dW is
    all-reduced after the second.  The micro-batch means are over the global count of each
    micro-batch, so the accumulated dW equals the mean of the two micro-batch oracle gradients
    on the union of the ranks' rows of that micro-batch."""
    split = 14
    res = _run(split, -1, buckets, 2)
    X, W, t = _data()
    N = X.shape[0]
    halves = [np.r_[0:7, split:split + (N - split) // 2],
              np.r_[7:split, split + (N - split) // 2:N]]
    ref_dW = np.zeros_like(W)
    for k, rows in enumerate(halves):
        f = oracle.forward_backward(X[rows], W, t[rows], VR, CAP, -1, g=0.5)
        ref_dW += f["dW"]
        for r in (0, 1):
            assert abs(res[r][1][k] - f["loss"]) < 1e-12
    for r in (0, 1):
        np.testing.assert_allclose(res[r][3], ref_dW, atol=1e-14)


def _rms_data(seed=3, N=30):
    X, W, t = _data(seed, N)
    rng = np.random.default_rng(seed + 100)
    H = rng.standard_normal((N, D)) * 2.0
    gamma = 1.0 + 0.2 * rng.standard_normal(D)
    return H, gamma, W, t


def _rms_worker(rank, world, store_path, split, q, micro=1):
    dist.init_process_group("gloo", init_method=f"file://{store_path}", rank=rank,
                            world_size=world)
    try:
        from lm_head_linear_gemm_b200.data_parallel import dp_step_rmsnorm
        H, gamma, W, t = _rms_data()
        lo, hi = (0, split) if rank == 0 else (split, H.shape[0])
        Hr, tr = torch.from_numpy(H[lo:hi].copy()), torch.from_numpy(t[lo:hi].copy())
        if micro == 1:
            loss, lse, dH, dg, dW, nv = dp_step_rmsnorm(Hr, torch.from_numpy(gamma),
                                                        torch.from_numpy(W), tr, VR, CAP, -1,
                                                        ops=OracleOps())
            q.put((rank, float(loss), dH.numpy(), dg.numpy(), dW.numpy(), int(nv.item())))
            return
        # this rank's rows as `micro` micro-batches, dgamma and dW accumulated with grad_scale
        # 1/micro and all-reduced after the last one
        cut = [(hi - lo) * k // micro for k in range(micro + 1)]
        dg = dW = None
        losses, dHs = [], []
        for k in range(micro):
            a, b = cut[k], cut[k + 1]
            loss, _, dH, dg, dW, nv = dp_step_rmsnorm(
                Hr[a:b], torch.from_numpy(gamma), torch.from_numpy(W), tr[a:b], VR, CAP, -1,
                ops=OracleOps(), dgamma=dg, dW=dW, accumulate=k > 0,
                allreduce_grads=k == micro - 1, grad_scale=1.0 / micro)
            losses.append(float(loss))
            dHs.append(dH.numpy())
        q.put((rank, losses, np.concatenate(dHs), dg.numpy(), dW.numpy(), int(nv.item())))
    finally:
        dist.destroy_process_group()


def _run_rms(split, micro=1):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    store_dir = tempfile.mkdtemp(prefix="flce_gloo_")
    procs = [ctx.Process(target=_rms_worker,
                         args=(r, 2, os.path.join(store_dir, "rendezvous"), split, q, micro))
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
    shutil.rmtree(store_dir, ignore_errors=True)
    return res


def test_two_rank_rmsnorm_accumulation_over_micro_batches():
    """Each rank's rows as two micro-batches with grad_scale 1/2, dgamma and dW accumulated and
    all-reduced after the second: they equal half the sum of the oracle's gradients of the two
    union micro-batches, whose losses both ranks hold."""
    split = 14
    res = _run_rms(split, micro=2)
    H, gamma, W, t = _rms_data()
    N = H.shape[0]
    half0 = split // 2
    half1 = split + (N - split) // 2
    halves = [np.r_[0:half0, split:half1], np.r_[half0:split, half1:N]]
    ref_dg, ref_dW = np.zeros_like(gamma), np.zeros_like(W)
    ref_dH = np.zeros_like(H)
    for k, rows in enumerate(halves):
        f = oracle.rmsnorm_head(H[rows], gamma, W, t[rows], VR, CAP, -1, g=0.5)
        ref_dg += f["dgamma"]
        ref_dW += f["dW"]
        ref_dH[rows] = f["dH"]
        for r in (0, 1):
            assert abs(res[r][1][k] - f["loss"]) < 1e-12
    for r in (0, 1):
        np.testing.assert_allclose(res[r][3], ref_dg, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(res[r][4], ref_dW, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(np.concatenate([res[0][2], res[1][2]]), ref_dH, rtol=1e-12,
                               atol=1e-14)


@pytest.mark.parametrize("split", [13, 4])
def test_two_rank_rmsnorm_step_equals_union_batch(split):
    """dp_step_rmsnorm on two gloo ranks: the global loss, dgamma and dW on both ranks and the
    ranks' dH rows equal one oracle step of the norm and the head on the union of their rows."""
    res = _run_rms(split)
    H, gamma, W, t = _rms_data()
    ref = oracle.rmsnorm_head(H, gamma, W, t, VR, CAP, -1)
    for r in (0, 1):
        assert abs(res[r][1] - ref["loss"]) < 1e-12
        np.testing.assert_allclose(res[r][3], ref["dgamma"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(res[r][4], ref["dW"], rtol=1e-12, atol=1e-14)
        assert res[r][5] == ref["n_valid"]
    np.testing.assert_allclose(np.concatenate([res[0][2], res[1][2]]), ref["dH"], rtol=1e-12,
                               atol=1e-14)
