"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same
seeded inputs.

Tolerances (fp32 accumulation of bf16 products, bf16 dX and gradient operand):
  |loss_gpu - loss_ref| <= 2e-3, max |lse_gpu - lse_ref| <= 2e-3,
  relL2(dX) <= 1e-2, relL2(dW) <= 1e-2,
plus a per-element guard (max error <= 5% of the tensor's max magnitude) so that a
single wrong tile cannot hide inside the L2 norm.  Small cases compare every element;
the full-size workloads, run in the launch configuration bench.py times, compare
sampled rows that the oracle computes one by one.
"""
import math

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

LOSS_TOL = 2e-3
LSE_TOL = 2e-3
REL_L2 = 1e-2


def _torch():
    import torch
    return torch


def to_dev(a_u16_or_i64):
    torch = _torch()
    a = np.ascontiguousarray(a_u16_or_i64)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def rel_l2(got, ref):
    den = np.linalg.norm(ref)
    return np.linalg.norm(got - ref) / (den if den > 0 else 1.0)


def check_tensor(name, got, ref, tol=REL_L2):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, name
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    r = rel_l2(got, ref)
    assert r <= tol, f"{name}: relL2 {r:.3e} > {tol}"
    scale = np.abs(ref).max()
    if scale > 0:
        worst = np.abs(got - ref).max()
        assert worst <= 0.05 * scale, f"{name}: max err {worst:.3e} vs max |ref| {scale:.3e}"
    return r


def run_gpu(inp, *, want_grads=True, chunk_rows=0, cap=None, recompute=False, g=None):
    import lm_head_linear_gemm_b200 as flce
    torch = _torch()
    c = inp["cfg"]
    cap = c.cap if cap is None else cap
    X, W, t = to_dev(inp["X"]), to_dev(inp["W"]), to_dev(inp["targets"])
    if recompute:
        loss, lse, _, _, ws = flce.forward(X, W, t, c.Vreal, cap, c.ignore_index, False,
                                           chunk_rows=chunk_rows)
        gt = None if g is None else torch.tensor(g, dtype=torch.float32, device="cuda")
        dX, dW = flce.backward(X, W, t, lse, c.Vreal, cap, c.ignore_index, grad_out=gt,
                               chunk_rows=chunk_rows)
    else:
        loss, lse, dX, dW, ws = flce.forward(X, W, t, c.Vreal, cap, c.ignore_index, want_grads,
                                             chunk_rows=chunk_rows)
    torch.cuda.synchronize()
    status, nv = flce.read_status(ws)
    out = dict(loss=float(loss.item()), lse=lse.double().cpu().numpy(), status=status, n_valid=nv)
    if dX is not None:
        out["dX"] = dX.double().cpu().numpy()
        out["dW"] = dW.double().cpu().numpy()
    return out


def oracle_full(inp, cap=None, g=1.0):
    c = inp["cfg"]
    cap = c.cap if cap is None else cap
    X = synth.bf16_to_f64(inp["X"])
    W = synth.bf16_to_f64(inp["W"])
    return oracle.forward_backward(X, W, inp["targets"], c.Vreal, cap, c.ignore_index, g)


def compare_full(got, ref, grads=True):
    assert abs(got["loss"] - ref["loss"]) <= LOSS_TOL, (got["loss"], ref["loss"])
    err = np.abs(got["lse"] - ref["lse"]).max() if len(ref["lse"]) else 0.0
    assert err <= LSE_TOL, f"lse max err {err:.3e}"
    assert got["n_valid"] == ref["n_valid"]
    if grads:
        check_tensor("dX", got["dX"], ref["dX"])
        check_tensor("dW", got["dW"], ref["dW"])


# ----------------------------------------------------------------------------- small, every element
def test_tiny_fused_and_recompute(cuda_device):
    inp = synth.make_inputs("tiny")
    ref = oracle_full(inp)
    got = run_gpu(inp)
    compare_full(got, ref)
    assert got["status"] == 0
    rec = run_gpu(inp, recompute=True)
    compare_full(rec, ref)
    c = inp["cfg"]
    assert np.abs(got["dW"][c.Vreal:]).max() == 0.0          # padded vocabulary rows


RAGGED = synth.custom_config("ragged", N=300, d=200, Vreal=1500, Vpad=1544, x_dist="normal",
                             w_std=0.05, target_dist="uniform", ignore_count=7)


@pytest.mark.parametrize("chunk_rows", [0, 128, 100])
def test_ragged_multi_tile(cuda_device, chunk_rows):
    """300 rows (3 row tiles, ragged), d = 200 (K tail), Vpad = 1544 (ragged vocabulary
    tile), chunks of 128 / 100 rows (ragged last chunk)."""
    inp = synth.make_inputs(RAGGED)
    ref = oracle_full(inp)
    compare_full(run_gpu(inp, chunk_rows=chunk_rows), ref)
    compare_full(run_gpu(inp, chunk_rows=chunk_rows, recompute=True), ref)


WIDE = synth.custom_config("wide", N=600, d=1024, Vreal=3000, Vpad=3008, x_dist="normal",
                           w_std=0.05, target_dist="uniform", ignore_count=9)


@pytest.mark.parametrize("chunk_rows", [0, 256])
def test_wide_dx_tiles_every_element(cuda_device, chunk_rows):
    """d = 1024: four 256-column blocks, so dX runs in wide tiles (two accumulators sharing
    each staged A' k-block); 600 rows give ragged row tiles and, with 256-row chunks, a ragged
    last chunk.  Every element of dX and dW against the oracle."""
    inp = synth.make_inputs(WIDE)
    ref = oracle_full(inp)
    compare_full(run_gpu(inp, chunk_rows=chunk_rows), ref)
    compare_full(run_gpu(inp, chunk_rows=chunk_rows, recompute=True), ref)


SUBLAUNCH = synth.custom_config("sublaunch", N=4200, d=128, Vreal=1000, Vpad=1024,
                                x_dist="normal", w_std=0.05, target_dist="uniform",
                                ignore_count=40)


@pytest.mark.parametrize("cap", [15.0, 0.0])
def test_logits_in_sub_launches_every_element(cuda_device, cap):
    """4200 rows in one chunk: the logits run as two launches (4096 rows + a ragged 104) that
    fill one chunk's partial sums and gradient operand; with and without the softcap (fixed
    reference vs (max, sum-exp) pairs).  Every element against the oracle."""
    inp = synth.make_inputs(SUBLAUNCH)
    ref = oracle_full(inp, cap=cap)
    compare_full(run_gpu(inp, cap=cap), ref)
    compare_full(run_gpu(inp, cap=cap, recompute=True), ref)
    stats = run_gpu(inp, cap=cap, want_grads=False)
    compare_full(stats, ref, grads=False)


@pytest.mark.parametrize("cap,w_std", [(0.0, 0.05), (2.0, 0.3), (50.0, 0.3), (15.0, 1.0)])
def test_softcap_variants(cuda_device, cap, w_std):
    """No softcap (online max path), a small cap (deep saturation), a large cap (softcap
    with the lse reference) and cap 15 with wide logits (|z| well beyond cap)."""
    c = synth.custom_config("cap", N=256, d=128, Vreal=900, Vpad=1024, x_dist="normal",
                            w_std=w_std, target_dist="uniform", ignore_count=3, cap=cap)
    inp = synth.make_inputs(c)
    ref = oracle_full(inp, cap=cap)
    compare_full(run_gpu(inp, cap=cap, chunk_rows=128), ref)
    compare_full(run_gpu(inp, cap=cap, recompute=True), ref)


@pytest.mark.parametrize("w_std,cap", [(2.0, 15.0), (0.05, 15.0), (1.0, 2.0)])
def test_softcap_math_tight(cuda_device, w_std, cap):
    """The epilogue's tanh / exp evaluation (two special-function exp2 and one special-function
    reciprocal per logit) against fp64 with a tolerance 10x tighter than the parity bar: with
    w_std = 2 the logits reach |z| ~ 80, far into the softcap's saturation; w_std = 0.05 keeps
    them near 0 where tanh is almost linear."""
    c = synth.custom_config("tight", N=256, d=128, Vreal=1000, Vpad=1024, x_dist="normal",
                            w_std=w_std, target_dist="uniform", ignore_count=2, cap=cap)
    inp = synth.make_inputs(c)
    ref = oracle_full(inp, cap=cap)
    got = run_gpu(inp, cap=cap)
    assert abs(got["loss"] - ref["loss"]) <= 2e-4
    assert np.abs(got["lse"] - ref["lse"]).max() <= 2e-4
    check_tensor("dX", got["dX"], ref["dX"], tol=REL_L2)
    check_tensor("dW", got["dW"], ref["dW"], tol=REL_L2)


def test_pages_vocabulary_every_element(cuda_device):
    """The pages' vocabulary (50257 -> 50304) and the small model's d = 1536, 512 rows."""
    inp = synth.make_inputs("small", N=512)
    ref = oracle_full(inp)
    got = run_gpu(inp)
    compare_full(got, ref)
    assert np.abs(got["dW"][50257:]).max() == 0.0
    compare_full(run_gpu(inp, recompute=True, chunk_rows=256), ref)


def test_bad_targets_are_ignored_and_flagged(cuda_device):
    inp = synth.make_inputs(RAGGED)
    t = inp["targets"].copy()
    t[5] = 1500          # a padded id: not a real token
    t[17] = 1_000_000
    t[40] = -3
    inp = dict(inp, targets=t)
    ref = oracle_full(inp)
    got = run_gpu(inp)
    assert got["status"] & 1
    compare_full(got, ref)
    assert np.abs(got["dX"][[5, 17, 40]]).max() == 0.0


def test_edge_cases(cuda_device):
    import lm_head_linear_gemm_b200 as flce
    torch = _torch()
    # one row
    inp = synth.make_inputs(synth.custom_config("one", 1, 64, 100, 128, w_std=0.1))
    compare_full(run_gpu(inp), oracle_full(inp))
    # no row in the loss: loss 0, zero gradients
    inp = synth.make_inputs(RAGGED)
    inp = dict(inp, targets=np.full(300, -1, np.int64))
    got = run_gpu(inp)
    assert got["loss"] == 0.0 and got["n_valid"] == 0
    assert np.abs(got["dX"]).max() == 0.0 and np.abs(got["dW"]).max() == 0.0
    # N = 0: loss 0, dW written as zeros (not accumulated)
    X = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.randn((128, 64), device="cuda").to(torch.bfloat16)
    t = torch.zeros((0,), dtype=torch.int64, device="cuda")
    dW = torch.full((128, 64), 7.0, device="cuda")
    loss, lse, dX, dW, _ = flce.forward(X, W, t, 100, 15.0, -1, True, dW=dW)
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and lse.numel() == 0 and float(dW.abs().max()) == 0.0


def test_smallest_hidden_and_vocabulary(cuda_device):
    """d = 8, the smallest hidden size the header allows (one 16-byte row: every tile is a K
    tail and a ragged N block), and Vpad = 40, a multiple of 8 but not of 16 (gradient-operand
    rows not 32-byte aligned), in one chunk and in chunks of 32 rows."""
    inp = synth.make_inputs(synth.custom_config("d8", 70, 8, 33, 40, w_std=0.5, ignore_count=3))
    ref = oracle_full(inp)
    for chunk_rows in (0, 32):
        got = run_gpu(inp, chunk_rows=chunk_rows)
        assert got["status"] == 0
        compare_full(got, ref)
    compare_full(run_gpu(inp, recompute=True), ref)


@pytest.mark.parametrize("ignore_index", [-100, 3])
def test_other_ignore_index(cuda_device, ignore_index):
    """ignore_index other than -1: PyTorch's default -100, and a vocabulary id (3), whose rows
    leave the loss while column 3 stays in every row's softmax.  Neither is a bad target."""
    cfg = synth.custom_config("ignore_other", N=300, d=200, Vreal=1500, Vpad=1544,
                              w_std=0.05, ignore_count=11, ignore_index=ignore_index)
    inp = synth.make_inputs(cfg)
    assert int(np.count_nonzero(inp["targets"] == ignore_index)) >= 11
    ref = oracle_full(inp)
    for chunk_rows in (0, 128):
        got = run_gpu(inp, chunk_rows=chunk_rows)
        assert got["status"] == 0
        compare_full(got, ref)


def test_accumulate_and_upstream_gradient(cuda_device):
    import lm_head_linear_gemm_b200 as flce
    torch = _torch()
    inp = synth.make_inputs(RAGGED)
    c = inp["cfg"]
    ref = oracle_full(inp)
    X, W, t = to_dev(inp["X"]), to_dev(inp["W"]), to_dev(inp["targets"])
    R = torch.randn(W.shape, device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    # fused forward accumulating onto R (gradient accumulation over micro-batches)
    _, _, _, dW, _ = flce.forward(X, W, t, c.Vreal, c.cap, -1, True, dW=R.clone(),
                                  accumulate_dW=True, chunk_rows=128)
    check_tensor("dW accumulated", (dW - R).double().cpu().numpy(), ref["dW"])
    # precomputed gradients scaled in place by g = 0.5
    _, _, dX, dW, _ = flce.forward(X, W, t, c.Vreal, c.cap, -1, True)
    flce.backward(X, W, t, None, c.Vreal, c.cap, -1, grad_out=torch.tensor(0.5, device="cuda"),
                  dX=dX, dW=dW, grads_precomputed=True)
    check_tensor("dX*g", dX.double().cpu().numpy(), 0.5 * ref["dX"])
    check_tensor("dW*g", dW.double().cpu().numpy(), 0.5 * ref["dW"])
    # recomputing backward with g = 2 accumulated onto R
    loss, lse, _, _, _ = flce.forward(X, W, t, c.Vreal, c.cap, -1, False)
    dX3, dW3 = flce.backward(X, W, t, lse, c.Vreal, c.cap, -1,
                             grad_out=torch.tensor(2.0, device="cuda"), dW=R.clone(),
                             accumulate_dW=True, chunk_rows=128)
    check_tensor("dX g=2", dX3.double().cpu().numpy(), 2 * ref["dX"])
    check_tensor("dW g=2 acc", (dW3 - R).double().cpu().numpy(), 2 * ref["dW"])


def test_compaction_across_chunks(cuda_device):
    """The gradient contractions run over each chunk's rows in the loss only.  Chunks of 256
    rows: the first keeps 192 rows (a whole number of 64-row k-blocks), the second none (its dW
    contribution is a zero tile added to the first chunk's), the last 88 of 88 (ragged).  Every
    element against the oracle, fused and recomputing; ignored rows have zero dX."""
    inp = synth.make_inputs(synth.custom_config("compact", N=600, d=200, Vreal=1500, Vpad=1544,
                                                x_dist="normal", w_std=0.05,
                                                target_dist="uniform", ignore_count=0))
    t = inp["targets"].copy()
    rng = np.random.default_rng(5)
    t[rng.permutation(256)[:64]] = -1
    t[256:512] = -1
    inp = dict(inp, targets=t)
    ref = oracle_full(inp)
    assert ref["n_valid"] == 192 + 88
    for recompute in (False, True):
        got = run_gpu(inp, chunk_rows=256, recompute=recompute)
        compare_full(got, ref)
        assert np.abs(got["dX"][t == -1]).max() == 0.0


def test_deterministic(cuda_device):
    inp = synth.make_inputs("small", N=640)
    a = run_gpu(inp, chunk_rows=256)
    b = run_gpu(inp, chunk_rows=256)
    assert a["loss"] == b["loss"]
    for k in ("lse", "dX", "dW"):
        assert np.array_equal(a[k], b[k]), k


def test_autograd_drop_in(cuda_device):
    import lm_head_linear_gemm_b200 as flce
    torch = _torch()
    inp = synth.make_inputs(RAGGED)
    c = inp["cfg"]
    ref = oracle_full(inp, g=3.0)
    X = to_dev(inp["X"]).requires_grad_(True)
    W = to_dev(inp["W"]).requires_grad_(True)
    t = to_dev(inp["targets"])
    loss = flce.fused_linear_cross_entropy(X, W, t, c.Vreal, c.cap, -1)
    (3.0 * loss).backward()
    assert abs(loss.item() - ref["loss"]) <= LOSS_TOL
    check_tensor("X.grad", X.grad.double().cpu().numpy(), ref["dX"])
    check_tensor("W.grad", W.grad.double().cpu().numpy(), ref["dW"])


# ----------------------------------------------------------------------------- full size, sampled
def _sampled_full_size(name, samples=48, seed=0):
    """The named workload at full size, default chunking (the bench's launch configuration).
    lse and dX are compared on sampled rows; dW on sampled vocabulary rows (random ones, all
    47 padded rows and the most frequent targets) using the oracle's lse of every row."""
    inp = synth.make_inputs(name)
    c = inp["cfg"]
    got = run_gpu(inp)
    assert got["status"] == 0
    X = synth.bf16_to_f64(inp["X"])
    W = synth.bf16_to_f64(inp["W"])
    t = inp["targets"]
    f = oracle.forward(X, W, t, c.Vreal, c.cap, c.ignore_index, block_rows=2048)
    assert abs(got["loss"] - f["loss"]) <= LOSS_TOL, (got["loss"], f["loss"])
    assert np.abs(got["lse"] - f["lse"]).max() <= LSE_TOL
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(c.N, samples, replace=False))
    dz = oracle.row_dlogits(X[rows], W, t[rows], f["lse"][rows], c.Vreal, c.cap, c.ignore_index,
                            f["n_valid"])
    check_tensor("dX rows", got["dX"][rows], dz @ W)
    counts = np.bincount(t[t >= 0], minlength=c.Vreal)
    frequent = np.argsort(-counts)[:16]
    vrows = np.unique(np.concatenate([rng.choice(c.Vreal, samples, replace=False), frequent,
                                      np.arange(c.Vreal, c.Vpad)]))
    ref_dW = oracle.dW_rows(X, W, t, f["lse"], vrows, c.Vreal, c.cap, c.ignore_index)
    check_tensor("dW rows", got["dW"][vrows], ref_dW)
    assert np.abs(got["dW"][c.Vreal:]).max() == 0.0
    return got, f


def test_full_size_small_model(cuda_device):
    _sampled_full_size("small")


def test_full_size_headline(cuda_device):
    got, f = _sampled_full_size("3.8b")
    assert math.isfinite(got["loss"])


def test_full_size_2k_context(cuda_device):
    """Batch 16 x context 2048 with W ~ N(0, 0.05): logits spread ~2.5x wider, more of them in
    the softcap's curved range."""
    got, f = _sampled_full_size("3.8b-2k")
    assert math.isfinite(got["loss"])


def test_rows_beyond_32bit_element_offsets(cuda_device):
    """N = 1400 x 512 = 716,800 rows at d = 3072: X and dX hold 2.2e9 elements each, past 32-bit
    element offsets, in 88 chunks (the last one half full) whose dW contributions accumulate.
    The rows are 1400 copies of a 512-row base problem (the 3.8b head's shapes and
    distributions), so the oracle on the base fixes every result: the loss and each row's lse
    equal the base's, each dX row is the base row's divided by 1400 (the count of rows in the
    loss is 1400 times larger), and dW equals the base's.  Copies of a row go through the same
    arithmetic, so they must agree bit for bit."""
    import lm_head_linear_gemm_b200 as flce
    torch = _torch()
    k = 1400
    inp = synth.make_inputs("3.8b", N=512)
    c = inp["cfg"]
    ref = oracle_full(inp)
    Xb, W, tb = to_dev(inp["X"]), to_dev(inp["W"]), to_dev(inp["targets"])
    X = Xb.repeat(k, 1)
    t = tb.repeat(k)
    assert X.numel() > 2**31
    loss, lse, dX, dW, ws = flce.forward(X, W, t, c.Vreal, c.cap, c.ignore_index, True)
    torch.cuda.synchronize()
    status, nv = flce.read_status(ws)
    assert status == 0 and nv == k * ref["n_valid"]
    del X
    assert abs(float(loss.item()) - ref["loss"]) <= LOSS_TOL
    lse_k = lse.view(k, 512)
    assert torch.equal(lse_k, lse_k[:1].expand(k, 512))
    assert np.abs(lse_k[0].double().cpu().numpy() - ref["lse"]).max() <= LSE_TOL
    dX_k = dX.view(k, 512, c.d)
    for i0 in range(0, k, 100):
        assert torch.equal(dX_k[i0:i0 + 100], dX_k[:1].expand(min(100, k - i0), 512, c.d)), i0
    check_tensor("dX rows (x copies)", dX_k[0].double().cpu().numpy() * k, ref["dX"])
    check_tensor("dW", dW.double().cpu().numpy(), ref["dW"])


def test_concurrent_calls_on_two_streams(cuda_device):
    """Calls on different streams with distinct workspaces are independent: issued back to
    back on two streams they give bit-identical results to the same calls run one by one."""
    import lm_head_linear_gemm_b200 as flce
    torch = _torch()
    a = synth.make_inputs(RAGGED)
    b = synth.make_inputs("small", N=700)
    dev = [(to_dev(x["X"]), to_dev(x["W"]), to_dev(x["targets"]), x["cfg"]) for x in (a, b)]

    def run(i, stream):
        X, W, t, c = dev[i]
        with torch.cuda.stream(stream):
            return flce.forward(X, W, t, c.Vreal, c.cap, -1, True, chunk_rows=128 * (i + 1),
                                stream=stream)

    s0, s1 = torch.cuda.Stream(), torch.cuda.Stream()
    seq = [run(0, s0), None]
    s0.synchronize()
    seq[1] = run(1, s0)
    s0.synchronize()
    par = [run(0, s0), run(1, s1)]
    torch.cuda.synchronize()
    for q, p in zip(seq, par):
        assert torch.equal(q[0], p[0]) and torch.equal(q[1], p[1])
        assert torch.equal(q[2], p[2]) and torch.equal(q[3], p[3])


def test_fused_step_captures_into_a_cuda_graph(cuda_device):
    """The library makes no synchronising or host-reading call on the launch path, so a fused
    forward + backward can be captured once and replayed; replays match eager results."""
    import lm_head_linear_gemm_b200 as flce
    torch = _torch()
    inp = synth.make_inputs(RAGGED)
    c = inp["cfg"]
    X, W, t = to_dev(inp["X"]), to_dev(inp["W"]), to_dev(inp["targets"])
    dX = torch.empty_like(X)
    dW = torch.empty(W.shape, dtype=torch.float32, device="cuda")
    g = torch.tensor(0.5, device="cuda")
    ws = flce.alloc_workspace(flce.make_shape(c.N, c.d, c.Vpad, c.Vreal, c.cap, -1, 128), True,
                              X.device)
    out = {}

    def step():
        loss, lse, _, _, _ = flce.forward(X, W, t, c.Vreal, c.cap, -1, True, dX=dX, dW=dW,
                                          workspace=ws, chunk_rows=128)
        flce.backward(X, W, t, lse, c.Vreal, c.cap, -1, grad_out=g, dX=dX, dW=dW,
                      grads_precomputed=True)
        out["loss"] = loss

    step()                                     # eager (also sets kernel attributes once)
    torch.cuda.synchronize()
    ref = (out["loss"].clone(), dX.clone(), dW.clone())
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    for _ in range(2):
        dX.zero_()
        dW.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out["loss"], ref[0])
        assert torch.equal(dX, ref[1]) and torch.equal(dW, ref[2])


def test_targets_in_the_padded_tail_tile(cuda_device):
    """Targets in the last real columns of the pages' vocabulary (50240..50256 share a 32-column
    epilogue chunk with padded columns; 50176.. is the half-padded last 256-column tile), the
    first column, and rows at chunk boundaries."""
    c = synth.custom_config("tail", N=260, d=128, Vreal=50257, Vpad=50304, x_dist="normal",
                            w_std=0.05, target_dist="uniform", ignore_count=0)
    inp = synth.make_inputs(c)
    t = inp["targets"].copy()
    special = [50256, 50255, 50240, 50239, 50176, 50175, 0, 1, 31, 32]
    t[:len(special)] = special
    t[127], t[128], t[255], t[256] = 50256, 50240, 0, 50255      # around 128-row chunk edges
    inp = dict(inp, targets=t)
    ref = oracle_full(inp)
    for chunk in (0, 128):
        got = run_gpu(inp, chunk_rows=chunk)
        compare_full(got, ref)
        assert np.abs(got["dW"][50257:]).max() == 0.0
        # the target rows of dW carry the -1 of the one-hot: check them element by element
        rows = np.array(sorted(set(special)))
        check_tensor("dW target rows", got["dW"][rows], ref["dW"][rows])
