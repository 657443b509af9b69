"""Gradient accumulation over micro-batches on the GPU, against the fp64 oracle.

The pages train with 7 gradient-accumulation micro-batches per optimizer step (config
appendix).  With each micro-batch's loss divided by 7 and the same number of rows in the loss
in every micro-batch, the accumulated head gradient equals the gradient of the mean loss over
the concatenated batch, which the oracle computes directly.  Covered: the fused C path
(``grad_scale`` = 1/7 with ``accumulate_dW``, fp32 and bf16 dW), and the autograd drop-in with an
fp32 ``main_grad`` (recomputing and hinted forms) and with plain bf16 W.grad accumulation.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

M = 7                       # micro-batches per optimizer step
ROWS = 300                  # rows per micro-batch
IGNORED = 7                 # rows with ignore_index in every micro-batch
REL_L2 = 1e-2
LOSS_TOL = 2e-3


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


@pytest.fixture(scope="module")
def batch():
    cfg = synth.custom_config("accum", N=M * ROWS, d=200, Vreal=1500, Vpad=1544,
                              x_dist="normal", w_std=0.05, target_dist="uniform", ignore_count=0)
    inp = synth.make_inputs(cfg)
    t = inp["targets"].copy()
    rng = np.random.default_rng(11)
    for m in range(M):
        t[m * ROWS + rng.permutation(ROWS)[:IGNORED]] = -1
    inp = dict(inp, targets=t)
    ref = oracle.forward_backward(synth.bf16_to_f64(inp["X"]), synth.bf16_to_f64(inp["W"]), t,
                                  cfg.Vreal, cfg.cap, -1)
    assert ref["n_valid"] == M * (ROWS - IGNORED)
    micro = []
    for m in range(M):
        sl = slice(m * ROWS, (m + 1) * ROWS)
        micro.append(oracle.forward(synth.bf16_to_f64(inp["X"][sl]),
                                    synth.bf16_to_f64(inp["W"]), t[sl], cfg.Vreal, cfg.cap, -1))
    return inp, ref, micro


def _slices():
    return [slice(m * ROWS, (m + 1) * ROWS) for m in range(M)]


@pytest.mark.parametrize("dw_dtype", ["float32", "bfloat16"])
def test_fused_path_accumulates_seven_micro_batches(cuda_device, batch, dw_dtype):
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp, ref, micro = batch
    c = inp["cfg"]
    X, W, t = _dev(inp["X"]), _dev(inp["W"]), _dev(inp["targets"])
    dW = torch.zeros(W.shape, dtype=getattr(torch, dw_dtype), device="cuda")
    g = torch.tensor(1.0 / M, dtype=torch.float32, device="cuda")
    dXs = []
    for m, sl in enumerate(_slices()):
        loss, _, dX, _, _ = flce.forward(X[sl].contiguous(), W, t[sl].contiguous(), c.Vreal,
                                         c.cap, -1, True, dW=dW, accumulate_dW=m > 0,
                                         grad_scale=g, chunk_rows=128)
        torch.cuda.synchronize()
        assert abs(loss.item() - micro[m]["loss"]) <= LOSS_TOL      # the loss is unscaled
        dXs.append(dX.double().cpu().numpy())
    assert _rel(np.concatenate(dXs), ref["dX"]) <= REL_L2
    assert _rel(dW.double().cpu().numpy(), ref["dW"]) <= REL_L2
    assert float(dW[c.Vreal:].abs().max()) == 0.0


def test_backward_refuses_to_scale_an_accumulated_dW(cuda_device, batch):
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp, _, _ = batch
    c = inp["cfg"]
    X, W, t = _dev(inp["X"][:ROWS]), _dev(inp["W"]), _dev(inp["targets"][:ROWS])
    _, lse, dX, dW, _ = flce.forward(X, W, t, c.Vreal, c.cap, -1, True)
    with pytest.raises(flce.FlceError):
        flce.backward(X, W, t, lse, c.Vreal, c.cap, -1, grad_out=torch.tensor(0.5, device="cuda"),
                      dX=dX, dW=dW, accumulate_dW=True, grads_precomputed=True)


@pytest.mark.parametrize("hint", [False, True])
def test_autograd_main_grad_accumulates_in_fp32(cuda_device, batch, hint):
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp, ref, micro = batch
    c = inp["cfg"]
    W = _dev(inp["W"]).requires_grad_(True)
    W.main_grad = torch.zeros(W.shape, dtype=torch.float32, device="cuda")
    t = _dev(inp["targets"])
    dXs = []
    for m, sl in enumerate(_slices()):
        X = _dev(inp["X"][sl]).requires_grad_(True)
        loss = flce.fused_linear_cross_entropy(X, W, t[sl].contiguous(), c.Vreal, c.cap, -1,
                                               grad_scale=(1.0 / M) if hint else None)
        (loss / M).backward()
        assert abs(loss.item() - micro[m]["loss"]) <= LOSS_TOL
        dXs.append(X.grad.double().cpu().numpy())
    torch.cuda.synchronize()
    assert W.grad is None                        # the gradient went to main_grad only
    assert _rel(np.concatenate(dXs), ref["dX"]) <= REL_L2
    assert _rel(W.main_grad.double().cpu().numpy(), ref["dW"]) <= REL_L2


def test_autograd_hint_mismatch_raises(cuda_device, batch):
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp, _, _ = batch
    c = inp["cfg"]
    W = _dev(inp["W"]).requires_grad_(True)
    W.main_grad = torch.zeros(W.shape, dtype=torch.float32, device="cuda")
    X = _dev(inp["X"][:ROWS]).requires_grad_(True)
    loss = flce.fused_linear_cross_entropy(X, W, _dev(inp["targets"][:ROWS]), c.Vreal, c.cap,
                                           -1, grad_scale=0.25)
    with pytest.raises(RuntimeError):
        (loss / 3).backward()


def test_autograd_bf16_weight_grad_accumulates(cuda_device, batch):
    """A plain bf16 head (no main_grad): dW is formed in bf16 and autograd adds the micro-batch
    gradients into W.grad in bf16, as bf16-master training does."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp, ref, _ = batch
    c = inp["cfg"]
    W = _dev(inp["W"]).requires_grad_(True)
    t = _dev(inp["targets"])
    for sl in _slices():
        X = _dev(inp["X"][sl]).requires_grad_(True)
        loss = flce.fused_linear_cross_entropy(X, W, t[sl].contiguous(), c.Vreal, c.cap, -1)
        (loss / M).backward()
    torch.cuda.synchronize()
    assert W.grad.dtype == torch.bfloat16
    assert _rel(W.grad.double().cpu().numpy(), ref["dW"]) <= REL_L2


def test_autograd_second_backward_raises(cuda_device, batch):
    """The gradients are formed in place: a second backward through the same graph must not
    scale them again."""
    import lm_head_linear_gemm_b200 as flce
    inp, _, _ = batch
    c = inp["cfg"]
    W = _dev(inp["W"]).requires_grad_(True)
    X = _dev(inp["X"][:ROWS]).requires_grad_(True)
    loss = flce.fused_linear_cross_entropy(X, W, _dev(inp["targets"][:ROWS]), c.Vreal, c.cap, -1)
    loss.backward(retain_graph=True)
    with pytest.raises(RuntimeError):
        loss.backward()
