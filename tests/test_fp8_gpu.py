"""GPU parity of the FP8 path: logits from e4m3 operands with tensorwise scales
(tcgen05 kind::f8f6f4); gradient contractions with the bf16 copies, or (grad_fp8) from an e5m2
gradient and the e4m3 operands.

* The device quantiser matches the reference encoder bit for bit (codes and scale).
* Kernel error: against the fp64 oracle evaluated on the dequantised e4m3 values for the
  logits and on the bf16 copies for the gradient products (or, with grad_fp8, the oracle's
  e5m2 gradient codes times the dequantised operands), with the ordinary parity bar.
* Quantisation error: against the all-bf16 oracle, reported and bounded loosely (three
  mantissa bits per logits operand, two per gradient code).
"""
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


def _rel(got, ref):
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def _run_fp8(inp, chunk_rows=0, want_grads=True, grad_fp8=False, **kw):
    import torch
    import lm_head_linear_gemm_b200 as flce
    c = inp["cfg"]
    sx = torch.tensor(float(inp["sX"]), dtype=torch.float32, device="cuda")
    sw = torch.tensor(float(inp["sW"]), dtype=torch.float32, device="cuda")
    X = None if grad_fp8 else _dev(inp["X"])
    W = None if grad_fp8 else _dev(inp["W"])
    loss, lse, dX, dW, ws = flce.forward_fp8(_dev(inp["X8"]), _dev(inp["W8"]), sx, sw, X, W,
                                             _dev(inp["targets"]), c.Vreal, c.cap,
                                             c.ignore_index, want_grads, chunk_rows=chunk_rows,
                                             grad_fp8=grad_fp8, **kw)
    torch.cuda.synchronize()
    status, nv = flce.read_status(ws)
    out = dict(loss=float(loss.item()), lse=lse.double().cpu().numpy(), status=status, n_valid=nv)
    if want_grads:
        out["dX"] = dX.double().cpu().numpy()
        out["dW"] = dW.double().cpu().numpy()
    return out


def _dequantised(inp):
    Xq = synth.e4m3_to_f64(inp["X8"]) * float(inp["sX"])
    Wq = synth.e4m3_to_f64(inp["W8"]) * float(inp["sW"])
    return Xq, Wq


def test_quantiser_matches_reference_encoder(cuda_device):
    import torch
    import lm_head_linear_gemm_b200 as flce
    inp = synth.make_fp8_inputs("small", N=1024)
    for key, skey in (("X", "sX"), ("W", "sW")):
        codes, scale = flce.quantize_e4m3(_dev(inp[key]))
        torch.cuda.synchronize()
        assert float(scale.item()) == float(inp[skey])
        assert np.array_equal(codes.cpu().numpy(), inp[key + "8"])


def test_fp8_against_dequantised_oracle(cuda_device):
    inp = synth.make_fp8_inputs("small", N=640)        # pages' vocabulary, d = 1536
    c = inp["cfg"]
    Xq, Wq = _dequantised(inp)
    ref = oracle.forward_backward(Xq, Wq, inp["targets"], c.Vreal, c.cap, c.ignore_index,
                                  Xg=synth.bf16_to_f64(inp["X"]), Wg=synth.bf16_to_f64(inp["W"]))
    for chunk in (0, 256):
        got = _run_fp8(inp, chunk_rows=chunk)
        assert got["status"] == 0 and got["n_valid"] == ref["n_valid"]
        assert abs(got["loss"] - ref["loss"]) <= LOSS_TOL
        assert np.abs(got["lse"] - ref["lse"]).max() <= LSE_TOL
        assert _rel(got["dX"], ref["dX"]) <= REL_L2
        assert _rel(got["dW"], ref["dW"]) <= REL_L2
        assert np.abs(got["dW"][c.Vreal:]).max() == 0.0
    stats = _run_fp8(inp, want_grads=False)
    assert abs(stats["loss"] - ref["loss"]) <= LOSS_TOL


def _check(name, got, ref, tol=REL_L2):
    r = _rel(got, ref)
    assert r <= tol, f"{name}: relL2 {r:.3e}"
    worst = np.abs(got - ref).max()
    assert worst <= 0.05 * np.abs(ref).max(), f"{name}: max err {worst:.3e}"
    return r


def test_fp8_gradients_against_quantisation_aware_oracle(cuda_device):
    """grad_fp8: e5m2 gradient codes times the e4m3 operands (kind::f8f6f4, e5m2 x e4m3), in one
    chunk and in 256-row chunks, against the oracle's FP8 gradient products; the loss and lse
    against the oracle on the dequantised operands.  Also accumulating with g = 0.5."""
    import torch
    inp = synth.make_fp8_inputs("small", N=640)        # pages' vocabulary, d = 1536
    c = inp["cfg"]
    Xq, Wq = _dequantised(inp)
    t = inp["targets"]
    f = oracle.forward(Xq, Wq, t, c.Vreal, c.cap, c.ignore_index)
    rX, rW = oracle.backward_fp8(Xq, Wq, t, c.Vreal, c.cap, c.ignore_index)
    for chunk in (0, 256):
        got = _run_fp8(inp, chunk_rows=chunk, grad_fp8=True)
        assert got["status"] == 0 and got["n_valid"] == f["n_valid"]
        assert abs(got["loss"] - f["loss"]) <= LOSS_TOL
        assert np.abs(got["lse"] - f["lse"]).max() <= LSE_TOL
        _check("dX", got["dX"], rX)
        _check("dW", got["dW"], rW)
        assert np.abs(got["dW"][c.Vreal:]).max() == 0.0
        assert np.abs(got["dX"][t == c.ignore_index]).max() == 0.0
    R = torch.randn((c.Vpad, c.d), device="cuda", generator=torch.Generator("cuda").manual_seed(2))
    acc = _run_fp8(inp, chunk_rows=256, grad_fp8=True, dW=R.clone(), accumulate_dW=True,
                   grad_scale=0.5)
    _check("dW accumulated, g = 0.5", acc["dW"] - R.double().cpu().numpy(), 0.5 * rW)
    _check("dX g = 0.5", acc["dX"], 0.5 * rX)
    bx, bw = oracle.backward(Xq, Wq, t, c.Vreal, c.cap, c.ignore_index,
                             Xg=synth.bf16_to_f64(inp["X"]), Wg=synth.bf16_to_f64(inp["W"]))
    print(f"fp8 gradients vs bf16-operand gradients: relL2 dX {_rel(got['dX'], bx):.2e}, "
          f"dW {_rel(got['dW'], bw):.2e}")


def test_fp8_bf16_dW_written_and_accumulated(cuda_device):
    """A bf16 dW from both gradient paths of the 8-bit workload (bf16 gradient products, and
    e5m2 x e4m3 products whose epilogue applies the tensorwise factor before the bf16 add):
    written by the first call with grad_scale 1/2, added to by the second, against the sum of
    the oracle's gradients."""
    import torch
    inp = synth.make_fp8_inputs("small", N=640)
    c = inp["cfg"]
    Xq, Wq = _dequantised(inp)
    t = inp["targets"]
    ref = oracle.forward_backward(Xq, Wq, t, c.Vreal, c.cap, c.ignore_index,
                                  Xg=synth.bf16_to_f64(inp["X"]), Wg=synth.bf16_to_f64(inp["W"]))
    _, rW8 = oracle.backward_fp8(Xq, Wq, t, c.Vreal, c.cap, c.ignore_index)
    for grad_fp8, rW in ((False, ref["dW"]), (True, rW8)):
        dW = torch.empty((c.Vpad, c.d), dtype=torch.bfloat16, device="cuda")
        for k in range(2):
            got = _run_fp8(inp, chunk_rows=256, grad_fp8=grad_fp8, dW=dW, accumulate_dW=k > 0,
                           grad_scale=0.5)
            assert got["status"] == 0
        _check(f"bf16 dW (grad_fp8={grad_fp8})", got["dW"], rW)
        assert np.abs(got["dW"][c.Vreal:]).max() == 0.0


RAGGED8 = synth.custom_config("fp8_ragged", N=300, d=208, Vreal=1500, Vpad=1544, w_std=0.05,
                              ignore_count=7)


@pytest.mark.parametrize("chunk_rows", [0, 128])
def test_fp8_ragged_shapes(cuda_device, chunk_rows):
    """300 rows (ragged row tiles), d = 208 (a K tail inside the second 128-byte k-block of the
    e4m3 operands, and ragged dX / dW column tiles), Vpad = 1544 (a ragged vocabulary tile and a
    K tail of the gradient operand), 7 ignored rows; one chunk and 128-row chunks; the bf16 and
    the FP8 gradient products, every element."""
    inp = synth.make_fp8_inputs(RAGGED8)
    c = inp["cfg"]
    Xq, Wq = _dequantised(inp)
    t = inp["targets"]
    ref = oracle.forward_backward(Xq, Wq, t, c.Vreal, c.cap, c.ignore_index,
                                  Xg=synth.bf16_to_f64(inp["X"]), Wg=synth.bf16_to_f64(inp["W"]))
    got = _run_fp8(inp, chunk_rows=chunk_rows)
    assert got["status"] == 0 and got["n_valid"] == ref["n_valid"]
    assert abs(got["loss"] - ref["loss"]) <= LOSS_TOL
    assert np.abs(got["lse"] - ref["lse"]).max() <= LSE_TOL
    _check("dX", got["dX"], ref["dX"])
    _check("dW", got["dW"], ref["dW"])
    rX, rW = oracle.backward_fp8(Xq, Wq, t, c.Vreal, c.cap, c.ignore_index)
    g8 = _run_fp8(inp, chunk_rows=chunk_rows, grad_fp8=True)
    assert g8["status"] == 0 and g8["loss"] == got["loss"]
    _check("dX (fp8 gradients)", g8["dX"], rX)
    _check("dW (fp8 gradients)", g8["dW"], rW)
    assert np.abs(g8["dW"][c.Vreal:]).max() == 0.0
    assert np.abs(g8["dX"][t == c.ignore_index]).max() == 0.0


@pytest.mark.parametrize("cap", [0.0, 50.0])
def test_fp8_logits_without_fixed_reference(cuda_device, cap):
    """No softcap, or a cap above 32: the e4m3 logits take the online-softmax statistics pass and
    the recompute of the gradient operand with lse, the scales applied to z (not folded into the
    exp2 argument as on the fixed-reference path); bf16 gradient products."""
    inp = synth.make_fp8_inputs(RAGGED8)
    c = inp["cfg"]
    Xq, Wq = _dequantised(inp)
    ref = oracle.forward_backward(Xq, Wq, inp["targets"], c.Vreal, cap, c.ignore_index,
                                  Xg=synth.bf16_to_f64(inp["X"]), Wg=synth.bf16_to_f64(inp["W"]))
    import dataclasses
    got = _run_fp8(dict(inp, cfg=dataclasses.replace(c, cap=cap)), chunk_rows=128)
    assert got["status"] == 0
    assert abs(got["loss"] - ref["loss"]) <= LOSS_TOL
    assert np.abs(got["lse"] - ref["lse"]).max() <= LSE_TOL
    _check("dX", got["dX"], ref["dX"])
    _check("dW", got["dW"], ref["dW"])


def test_fp8_quantisation_error_against_bf16_oracle(cuda_device):
    """Reported figure: how far e4m3 logits move the loss and gradients from the bf16 result."""
    inp = synth.make_fp8_inputs("small", N=640)
    c = inp["cfg"]
    ref = oracle.forward_backward(synth.bf16_to_f64(inp["X"]), synth.bf16_to_f64(inp["W"]),
                                  inp["targets"], c.Vreal, c.cap, c.ignore_index)
    got = _run_fp8(inp)
    dloss = abs(got["loss"] - ref["loss"])
    rx, rw = _rel(got["dX"], ref["dX"]), _rel(got["dW"], ref["dW"])
    print(f"fp8 vs bf16 oracle: |dloss| {dloss:.2e}, max|dlse| "
          f"{np.abs(got['lse'] - ref['lse']).max():.2e}, relL2 dX {rx:.2e}, dW {rw:.2e}")
    assert dloss <= 5e-2 and rx <= 0.2 and rw <= 0.2


def test_fp8_full_size_sampled(cuda_device):
    """The large micro-batch workload (N = 65536, 5% ignored) in the bench's launch
    configuration: loss and lse on all rows, dX on sampled rows, dW on sampled vocabulary
    rows (random, the most frequent targets and all padded rows), against the oracle on the
    dequantised logits operands and the bf16 gradient operands."""
    inp = synth.make_fp8_inputs("fp8")
    c = inp["cfg"]
    got = _run_fp8(inp)
    assert got["status"] == 0
    Xq, Wq = _dequantised(inp)
    Xb = synth.bf16_to_f64(inp["X"])
    Wb = synth.bf16_to_f64(inp["W"])
    t = inp["targets"]
    f = oracle.forward(Xq, Wq, t, c.Vreal, c.cap, c.ignore_index, block_rows=2048)
    assert abs(got["loss"] - f["loss"]) <= LOSS_TOL
    assert np.abs(got["lse"] - f["lse"]).max() <= LSE_TOL
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(c.N, 32, replace=False))
    dz = oracle.row_dlogits(Xq[rows], Wq, t[rows], f["lse"][rows], c.Vreal, c.cap,
                            c.ignore_index, f["n_valid"])
    assert _rel(got["dX"][rows], dz @ Wb) <= REL_L2
    counts = np.bincount(t[t >= 0], minlength=c.Vreal)
    vrows = np.unique(np.concatenate([rng.choice(c.Vreal, 24, replace=False),
                                      np.argsort(-counts)[:8], np.arange(c.Vreal, c.Vpad)]))
    ref_dW = oracle.dW_rows(Xq, Wq, t, f["lse"], vrows, c.Vreal, c.cap, c.ignore_index, Xg=Xb)
    assert _rel(got["dW"][vrows], ref_dW) <= REL_L2
    assert np.abs(got["dW"][c.Vreal:]).max() == 0.0
    # quantisation error at full size (reported): the sampled rows against the all-bf16 oracle
    lse_b, _, _ = oracle.row_forward(Xb[rows], Wb, t[rows], c.Vreal, c.cap, c.ignore_index)
    dz_b = oracle.row_dlogits(Xb[rows], Wb, t[rows], lse_b, c.Vreal, c.cap, c.ignore_index,
                              f["n_valid"])
    e_lse = np.abs(got["lse"][rows] - lse_b).max()
    e_dx = _rel(got["dX"][rows], dz_b @ Wb)
    print(f"fp8 N=65536 vs bf16 oracle on {len(rows)} rows: max|dlse| {e_lse:.2e}, "
          f"relL2 dX {e_dx:.2e}; vs dequantised oracle: max|dlse| "
          f"{np.abs(got['lse'][rows] - f['lse'][rows]).max():.2e}, relL2 dX "
          f"{_rel(got['dX'][rows], dz @ Wb):.2e}")
    assert e_lse <= 5e-2 and e_dx <= 0.2
    # the same workload with the gradient contractions in FP8 (e5m2 x e4m3)
    g8 = _run_fp8(inp, grad_fp8=True)
    assert g8["status"] == 0 and g8["loss"] == got["loss"]
    scale = 1.0 / (f["n_valid"] * oracle.E5M2_SCALE)
    q = oracle.dlogits_e5m2(Xq[rows], Wq, t[rows], c.Vreal, c.cap, c.ignore_index)
    _check("fp8 dX rows", g8["dX"][rows], scale * (q @ Wq))
    ref_dW8 = oracle.dW_rows_fp8(Xq, Wq, t, f["lse"], vrows, c.Vreal, c.cap, c.ignore_index)
    _check("fp8 dW rows", g8["dW"][vrows], ref_dW8)
    print(f"fp8 gradients N=65536 vs bf16 oracle on {len(rows)} rows: relL2 dX "
          f"{_rel(g8['dX'][rows], dz_b @ Wb):.2e}")
