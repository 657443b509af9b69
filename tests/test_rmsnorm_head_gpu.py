"""The final RMSNorm and the head in one call (flce_forward_rmsnorm) against the fp64 oracle
(oracle.rmsnorm_head: x = rmsnorm(h) rounded to bf16, the head on x, the chain rule through the
norm with the exact rows).

With 0 < cap <= 32 the norm's backward is folded into the dX contraction (the epilogue writes
dH; dgamma from per-32-row partials), otherwise dX goes through a buffer and the separate row
kernels.  Small shapes compare every element of loss, lse, dH, dgamma and dW; the 3.8b head's
width (d = 3072, Vpad = 50304) runs with 1024 rows, every element, and at the headline's 16384
rows in its default chunking on sampled rows.  Tolerances as for the head alone (fp32
accumulation of bf16 products, bf16 dH): loss and lse within 2e-3, relative L2 within 1e-2 with
a per-element guard of 5% of the tensor's largest magnitude.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

LOSS_TOL = 2e-3
LSE_TOL = 2e-3
REL_L2 = 1e-2
EPS = 1e-6


def _dev(bits):
    import torch
    a = np.ascontiguousarray(bits)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _rel(got, ref):
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def _check(name, got, ref, tol=REL_L2):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, name
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    r = _rel(got, ref)
    assert r <= tol, f"{name}: relL2 {r:.3e}"
    scale = np.abs(ref).max()
    if scale > 0:
        assert np.abs(got - ref).max() <= 0.05 * scale, name


def _run(inp, chunk_rows=0, cap=None, g=None, dgamma=None, dW=None, accumulate=False):
    import torch
    import lm_head_linear_gemm_b200 as flce
    c = inp["cfg"]
    cap = c.cap if cap is None else cap
    loss, lse, dH, dg, dW_, ws = flce.forward_rmsnorm(
        _dev(inp["H"]), _dev(inp["gamma"]), _dev(inp["W"]), _dev(inp["targets"]), c.Vreal, cap,
        c.ignore_index, EPS, want_grads=True, dgamma=dgamma, dW=dW, accumulate=accumulate,
        chunk_rows=chunk_rows, grad_scale=g)
    torch.cuda.synchronize()
    status, nv = flce.read_status(ws)
    return dict(loss=float(loss.item()), lse=lse.double().cpu().numpy(), status=status,
                n_valid=nv, dH=dH.double().cpu().numpy(), dgamma=dg.double().cpu().numpy(),
                dW=dW_.double().cpu().numpy(), dg_t=dg, dW_t=dW_)


def _oracle(inp, cap=None, g=1.0):
    c = inp["cfg"]
    cap = c.cap if cap is None else cap
    return oracle.rmsnorm_head(synth.bf16_to_f64(inp["H"]), synth.bf16_to_f64(inp["gamma"]),
                               synth.bf16_to_f64(inp["W"]), inp["targets"], c.Vreal, cap,
                               c.ignore_index, EPS, g)


def _compare(got, ref, grads=("dH", "dgamma", "dW")):
    assert got["status"] == 0
    assert got["n_valid"] == ref["n_valid"]
    assert abs(got["loss"] - ref["loss"]) <= LOSS_TOL, (got["loss"], ref["loss"])
    assert np.abs(got["lse"] - ref["lse"]).max() <= LSE_TOL
    for k in grads:
        _check(k, got[k], ref[k])


RAGGED = synth.custom_config("rms_ragged", N=300, d=200, Vreal=1500, Vpad=1544, w_std=0.1,
                             ignore_count=7)


@pytest.mark.parametrize("chunk_rows", [0, 128, 100])
def test_fold_every_element(cuda_device, chunk_rows):
    """300 rows (ragged row tiles; with 128 / 100-row chunks several chunks, a ragged last one,
    and dgamma summed over chunks), d = 200 (a K tail, and dH / dgamma columns in a partial
    tile), Vpad = 1544 (ragged vocabulary tile), 7 ignored rows (compacted away)."""
    inp = synth.make_rmsnorm_inputs(RAGGED)
    ref = _oracle(inp)
    got = _run(inp, chunk_rows=chunk_rows)
    _compare(got, ref)
    ignored = inp["targets"] == -1
    assert np.abs(got["dH"][ignored]).max() == 0.0           # rows outside the loss
    assert np.abs(got["dW"][RAGGED.Vreal:]).max() == 0.0     # padded vocabulary rows


WIDE = synth.custom_config("rms_wide", N=600, d=1024, Vreal=3000, Vpad=3008, w_std=0.05,
                           ignore_count=9)


def test_fold_in_wide_dx_tiles(cuda_device):
    """d = 1024: the dX contraction runs in wide tiles (two accumulators), so each epilogue
    call folds half of a 512-column block; 600 rows in 256-row chunks."""
    inp = synth.make_rmsnorm_inputs(WIDE)
    _compare(_run(inp, chunk_rows=256), _oracle(inp))


@pytest.mark.parametrize("cap", [0.0, 40.0])
def test_separate_backward_without_fixed_reference(cuda_device, cap):
    """No softcap, or a cap above 32: dX through the workspace, then the RMSNorm row kernels."""
    inp = synth.make_rmsnorm_inputs(RAGGED)
    _compare(_run(inp, chunk_rows=128, cap=cap), _oracle(inp, cap=cap))


def test_accumulate_with_upstream_gradient(cuda_device):
    """Two micro-batches with g = 1/2 into one dgamma and one dW (accumulate on the second):
    the sums equal half the sum of the two oracle gradients; dH is each call's own."""
    import torch
    a = synth.make_rmsnorm_inputs(RAGGED, seed=1)
    b = synth.make_rmsnorm_inputs(RAGGED, seed=2)
    b["W"], b["gamma"] = a["W"], a["gamma"]
    ga = _run(a, g=0.5)
    gb = _run(b, g=0.5, dgamma=ga["dg_t"], dW=ga["dW_t"], accumulate=True)
    ra, rb = _oracle(a, g=0.5), _oracle(b, g=0.5)
    _check("dH (first)", ga["dH"], ra["dH"])
    _check("dH (second)", gb["dH"], rb["dH"])
    _check("dgamma", gb["dgamma"], ra["dgamma"] + rb["dgamma"])
    _check("dW", gb["dW"], ra["dW"] + rb["dW"])
    assert torch.equal(gb["dg_t"], ga["dg_t"])                # accumulated in place


def test_deterministic(cuda_device):
    inp = synth.make_rmsnorm_inputs(WIDE)
    a, b = _run(inp, chunk_rows=256), _run(inp, chunk_rows=256)
    for k in ("lse", "dH", "dgamma", "dW"):
        np.testing.assert_array_equal(a[k], b[k])
    assert a["loss"] == b["loss"]


def test_autograd_drop_in(cuda_device):
    """fused_rmsnorm_linear_cross_entropy: loss * 3 backward gives the oracle's gradients of
    3 * loss in H.grad, gamma.grad and W.grad (all bf16 leaves)."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp = synth.make_rmsnorm_inputs(RAGGED)
    c = inp["cfg"]
    H = _dev(inp["H"]).requires_grad_(True)
    gamma = _dev(inp["gamma"]).requires_grad_(True)
    W = _dev(inp["W"]).requires_grad_(True)
    t = _dev(inp["targets"])
    loss = flce.fused_rmsnorm_linear_cross_entropy(H, gamma, W, t, c.Vreal, c.cap, -1, EPS)
    (loss * 3.0).backward()
    torch.cuda.synchronize()
    ref = _oracle(inp, g=3.0)
    assert abs(float(loss.item()) - ref["loss"]) <= LOSS_TOL
    assert gamma.grad.dtype == torch.bfloat16
    _check("H.grad", H.grad.double().cpu().numpy(), ref["dH"])
    _check("gamma.grad", gamma.grad.double().cpu().numpy(), ref["dgamma"])
    _check("W.grad", W.grad.double().cpu().numpy(), ref["dW"])
    with pytest.raises(RuntimeError):
        loss2 = flce.fused_rmsnorm_linear_cross_entropy(H, gamma, W, t, c.Vreal, c.cap, -1, EPS)
        loss2.backward(retain_graph=True)
        loss2.backward()


def test_headline_width_every_element(cuda_device):
    """The 3.8b head's width (d = 3072, Vpad = 50304, Zipf targets, 2% ignored) with 1024 rows:
    every element of dH, dgamma and dW against the full oracle."""
    inp = synth.make_rmsnorm_inputs("3.8b", N=1024)
    _compare(_run(inp), _oracle(inp))


def test_headline_sampled(cuda_device):
    """The headline's 16384 rows in the default chunking (two 8192-row chunks, compacted):
    loss and every lse against the oracle's forward, dH on sampled rows (the oracle's dX rows
    through the norm's chain rule, which is row-local), dW on sampled vocabulary rows."""
    inp = synth.make_rmsnorm_inputs("3.8b")
    c = inp["cfg"]
    got = _run(inp)
    assert got["status"] == 0
    H = synth.bf16_to_f64(inp["H"])
    gamma = synth.bf16_to_f64(inp["gamma"])
    W = synth.bf16_to_f64(inp["W"])
    t = inp["targets"]
    x = oracle.round_bf16(oracle.rmsnorm_forward(H, gamma, EPS)[0])
    f = oracle.forward(x, W, t, c.Vreal, c.cap, c.ignore_index, block_rows=2048)
    assert abs(got["loss"] - f["loss"]) <= LOSS_TOL
    assert np.abs(got["lse"] - f["lse"]).max() <= LSE_TOL
    rng = np.random.default_rng(3)
    rows = np.sort(np.concatenate([rng.choice(c.N, 24, replace=False),
                                   np.nonzero(t == c.ignore_index)[0][:4]]))
    dz = oracle.row_dlogits(x[rows], W, t[rows], f["lse"][rows], c.Vreal, c.cap,
                            c.ignore_index, f["n_valid"])
    dH_ref, _ = oracle.rmsnorm_backward(H[rows], gamma, dz @ W, EPS)
    _check("dH rows", got["dH"][rows], dH_ref)
    counts = np.bincount(t[t >= 0], minlength=c.Vreal)
    vrows = np.unique(np.concatenate([rng.choice(c.Vreal, 16, replace=False),
                                      np.argsort(-counts)[:8], np.arange(c.Vreal, c.Vpad)]))
    ref_dW = oracle.dW_rows(x, W, t, f["lse"], vrows, c.Vreal, c.cap, c.ignore_index)
    _check("dW rows", got["dW"][vrows], ref_dW)


def test_edge_cases(cuda_device):
    """Loss only (lse against the oracle's forward); every row ignored (loss 0, zero gradients,
    dgamma written as zeros); a bad target (flagged, treated as ignored); N = 0 (dgamma and dW
    written as zeros, or left as they are when accumulating)."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp = synth.make_rmsnorm_inputs(RAGGED)
    c = inp["cfg"]
    H, gamma, W = _dev(inp["H"]), _dev(inp["gamma"]), _dev(inp["W"])
    # loss and lse only
    loss, lse, dH, dg, dW, _ = flce.forward_rmsnorm(H, gamma, W, _dev(inp["targets"]), c.Vreal,
                                                    c.cap, c.ignore_index, EPS)
    torch.cuda.synchronize()
    assert dH is None and dg is None and dW is None
    ref = _oracle(inp)
    assert abs(float(loss.item()) - ref["loss"]) <= LOSS_TOL
    assert np.abs(lse.double().cpu().numpy() - ref["lse"]).max() <= LSE_TOL
    # every row ignored
    got = _run(dict(inp, targets=np.full(c.N, -1, np.int64)))
    assert got["loss"] == 0.0 and got["n_valid"] == 0 and got["status"] == 0
    for k in ("dH", "dgamma", "dW"):
        assert np.abs(got[k]).max() == 0.0, k
    # a bad target: flagged and treated as ignored
    t = inp["targets"].copy()
    t[5] = c.Vreal + 3
    bad = dict(inp, targets=t)
    got = _run(bad)
    assert got["status"] & flce.DEV_BAD_TARGET
    t_ref = t.copy()
    t_ref[5] = -1
    _compare(dict(got, status=0), _oracle(dict(inp, targets=t_ref)))
    # N = 0
    H0 = torch.zeros((0, c.d), dtype=torch.bfloat16, device="cuda")
    t0 = torch.zeros((0,), dtype=torch.int64, device="cuda")
    dg0 = torch.full((c.d,), 7.0, device="cuda")
    dW0 = torch.full((c.Vpad, c.d), 7.0, device="cuda")
    loss, lse, _, dg0, dW0, _ = flce.forward_rmsnorm(H0, gamma, W, t0, c.Vreal, c.cap, -1, EPS,
                                                     want_grads=True, dgamma=dg0, dW=dW0)
    torch.cuda.synchronize()
    assert float(loss.item()) == 0.0 and lse.numel() == 0
    assert float(dg0.abs().max()) == 0.0 and float(dW0.abs().max()) == 0.0
    dg1 = torch.full((c.d,), 7.0, device="cuda")
    dW1 = torch.full((c.Vpad, c.d), 7.0, device="cuda")
    flce.forward_rmsnorm(H0, gamma, W, t0, c.Vreal, c.cap, -1, EPS, want_grads=True, dgamma=dg1,
                         dW=dW1, accumulate=True)
    torch.cuda.synchronize()
    assert float(dg1.min()) == 7.0 and float(dg1.max()) == 7.0
    assert float(dW1.min()) == 7.0 and float(dW1.max()) == 7.0


def test_one_call_captures_into_a_cuda_graph(cuda_device):
    """The one-call path launches without synchronising or reading on the host, so a training
    step of the norm and the head (forward, then the upstream gradient applied) can be captured
    once and replayed; replays match the eager results bit for bit."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp = synth.make_rmsnorm_inputs(RAGGED)
    c = inp["cfg"]
    H, gamma, W, t = _dev(inp["H"]), _dev(inp["gamma"]), _dev(inp["W"]), _dev(inp["targets"])
    dH = torch.empty_like(H)
    dg = torch.empty(c.d, dtype=torch.float32, device="cuda")
    dW = torch.empty(W.shape, dtype=torch.float32, device="cuda")
    g = torch.tensor(0.5, device="cuda")
    import ctypes
    shape = flce.make_shape(c.N, c.d, c.Vpad, c.Vreal, c.cap, -1, 128)
    ws = torch.empty(int(flce.lib().flce_workspace_bytes_rmsnorm(ctypes.byref(shape), 1)),
                     dtype=torch.uint8, device="cuda")
    out = {}

    def step():
        loss, _, _, _, _, _ = flce.forward_rmsnorm(H, gamma, W, t, c.Vreal, c.cap, -1, EPS, True,
                                                   dH=dH, dgamma=dg, dW=dW, workspace=ws,
                                                   chunk_rows=128)
        flce.scale_grads_rmsnorm(g, dH, dg, dW, c.Vreal, c.cap, -1)
        out["loss"] = loss

    step()
    torch.cuda.synchronize()
    ref = (out["loss"].clone(), dH.clone(), dg.clone(), dW.clone())
    _check("dH of g * loss", dH.double().cpu().numpy(), _oracle(inp, g=0.5)["dH"])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    for _ in range(2):
        for b in (dH, dg, dW):
            b.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out["loss"], ref[0])
        assert torch.equal(dH, ref[1]) and torch.equal(dg, ref[2]) and torch.equal(dW, ref[3])


def test_one_call_beyond_32bit_element_offsets(cuda_device):
    """N = 1400 x 512 = 716,800 rows at d = 3072: H, the normalised rows and dH hold 2.2e9
    elements each, past 32-bit element offsets, in 88 chunks whose dgamma and dW contributions
    accumulate.  The rows are 1400 copies of a 512-row base problem, so the oracle on the base
    fixes every result: the loss and each row's lse equal the base's, each dH row is the base
    row's divided by 1400 (1400 times as many rows in the loss), and dgamma and dW equal the
    base's.  Copies of a row go through the same arithmetic and must agree bit for bit."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    k = 1400
    inp = synth.make_rmsnorm_inputs("3.8b", N=512)
    c = inp["cfg"]
    ref = _oracle(inp)
    H = _dev(inp["H"]).repeat(k, 1)
    t = _dev(inp["targets"]).repeat(k)
    assert H.numel() > 2**31
    loss, lse, dH, dg, dW, ws = flce.forward_rmsnorm(H, _dev(inp["gamma"]), _dev(inp["W"]), t,
                                                     c.Vreal, c.cap, c.ignore_index, EPS, True)
    torch.cuda.synchronize()
    status, nv = flce.read_status(ws)
    assert status == 0 and nv == k * ref["n_valid"]
    del H, ws
    assert abs(float(loss.item()) - ref["loss"]) <= LOSS_TOL
    lse_k = lse.view(k, 512)
    assert torch.equal(lse_k, lse_k[:1].expand(k, 512))
    assert np.abs(lse_k[0].double().cpu().numpy() - ref["lse"]).max() <= LSE_TOL
    dH_k = dH.view(k, 512, c.d)
    for i0 in range(0, k, 100):
        assert torch.equal(dH_k[i0:i0 + 100], dH_k[:1].expand(min(100, k - i0), 512, c.d)), i0
    _check("dH rows (x copies)", dH_k[0].double().cpu().numpy() * k, ref["dH"])
    _check("dgamma", dg.double().cpu().numpy(), ref["dgamma"])
    _check("dW", dW.double().cpu().numpy(), ref["dW"])
