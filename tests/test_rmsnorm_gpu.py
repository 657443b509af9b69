"""The final RMSNorm in front of the head: forward (x, rstd), backward (dH, dgamma) and the
chain rmsnorm -> fused linear cross-entropy through autograd, against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


def _bf16(a):
    import torch
    return torch.from_numpy(synth.f32_to_bf16_bits(np.asarray(a, np.float32)).view(np.int16)).view(
        torch.bfloat16).cuda()


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def test_rmsnorm_forward_backward(cuda_device):
    import torch
    import lm_head_linear_gemm_b200 as flce
    rng = np.random.default_rng(2)
    N, d = 333, 1536
    Hb = _bf16(rng.standard_normal((N, d)) * 3.0)
    gb = _bf16(1.0 + 0.2 * rng.standard_normal(d))
    dXb = _bf16(rng.standard_normal((N, d)) * 1e-3)
    H = Hb.double().cpu().numpy()
    g = gb.double().cpu().numpy()
    dX = dXb.double().cpu().numpy()
    X, rstd = flce.rmsnorm_forward(Hb, gb, 1e-6)
    dH, dgamma = flce.rmsnorm_backward(Hb, gb, rstd, dXb)
    dgamma2 = dgamma.clone()
    flce.rmsnorm_backward(Hb, gb, rstd, dXb, dgamma=dgamma2, accumulate_dgamma=True)
    torch.cuda.synchronize()
    xr, rr = oracle.rmsnorm_forward(H, g, 1e-6)
    dHr, dgr = oracle.rmsnorm_backward(H, g, dX, 1e-6)
    assert np.abs(rstd.double().cpu().numpy() - rr).max() <= 1e-5 * rr.max()
    assert _rel(X.double().cpu().numpy(), xr) <= 5e-3
    assert _rel(dH.double().cpu().numpy(), dHr) <= 1e-2
    assert _rel(dgamma.double().cpu().numpy(), dgr) <= 1e-4
    assert _rel(dgamma2.double().cpu().numpy(), 2 * dgr) <= 1e-4


def test_rmsnorm_then_fused_loss_autograd(cuda_device):
    import torch
    import lm_head_linear_gemm_b200 as flce
    rng = np.random.default_rng(4)
    cfg = synth.custom_config("rms", N=300, d=256, Vreal=1500, Vpad=1544, w_std=0.1,
                              ignore_count=5)
    inp = synth.make_inputs(cfg)
    Hn = rng.standard_normal((cfg.N, cfg.d)) * 2.0
    gn = 1.0 + 0.2 * rng.standard_normal(cfg.d)
    Hb = _bf16(Hn).requires_grad_(True)
    gb = _bf16(gn).requires_grad_(True)
    W = torch.from_numpy(inp["W"].view(np.int16)).view(torch.bfloat16).cuda().requires_grad_(True)
    t = torch.from_numpy(inp["targets"]).cuda()
    x = flce.rmsnorm(Hb, gb, 1e-6)
    loss = flce.fused_linear_cross_entropy(x, W, t, cfg.Vreal, cfg.cap, -1)
    loss.backward()
    H = Hb.detach().double().cpu().numpy()
    g = gb.detach().double().cpu().numpy()
    Wd = W.detach().double().cpu().numpy()
    # reference chain on the same bf16 rounding point: x rounded to bf16 as the kernel does
    xr, _ = oracle.rmsnorm_forward(H, g, 1e-6)
    xr_b = synth.bf16_to_f64(synth.f32_to_bf16_bits(xr.astype(np.float32)))
    f = oracle.forward_backward(xr_b, Wd, inp["targets"], cfg.Vreal, cfg.cap, -1)
    dHr, dgr = oracle.rmsnorm_backward(H, g, f["dX"], 1e-6)
    assert abs(loss.item() - f["loss"]) <= 2e-3
    assert _rel(Hb.grad.double().cpu().numpy(), dHr) <= 1e-2
    assert _rel(gb.grad.double().cpu().numpy(), dgr) <= 1e-2
    assert _rel(W.grad.double().cpu().numpy(), f["dW"]) <= 1e-2
