"""fp64 CPU oracle for the fused LM-head linear + softcapped cross-entropy.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``lm_head_linear_gemm_b200``) never imports it and
shares no code with it.

What it computes is the plain definition, written out in float64 on bf16-rounded
inputs (the GPU path reads the same bf16 values):

* logits of the untied LM head, ``z = X W^T`` over all ``Vpad`` rows of ``W``
  (little-lm 3.8B write-up, "Setup": LM head of 154.5M = 50304 x 3072 parameters);
* the logit softcap ``s = cap * tanh(z / cap)`` with ``cap = 15`` (the config appendix sets a
  logit softcap of 15 and passes the same value to its third-party fused loss).
  The pages name the softcap but print no formula; ``cap*tanh(z/cap)`` is the
  reading adopted.  ``cap <= 0`` means no softcap (``s = z``);
* the padded vocabulary (50257 real tokens padded to 50304 for the tensor cores,
  "Increasing throughput" / vocabulary padding): padded columns ``j >= Vreal``
  take no part in the softmax;
* cross entropy averaged over the positions whose target is not ``ignore_index``
  (the pages state neither an ignore index nor a reduction; mean over valid rows
  is the reading adopted; with no valid row the loss is 0);
* analytic gradients ``dX = dz W`` and ``dW = dz^T X`` with
  ``dz = g/Nv * (softmax(s) - onehot(t)) * (1 - tanh^2(z/cap))``.
* FP8 variant (the write-ups train with FP8 GEMMs under dynamic tensorwise scaling,
  "Increasing throughput"): the logits come from the e4m3 operands times their scales while
  the two gradient products use the bf16 copies -- ``backward(..., Xg=, Wg=)``; or, with FP8
  gradient products too (the write-ups' "three GEMMs in FP8": one forward, two backward),
  ``backward_fp8`` -- the softmax gradient is encoded in e5m2 and multiplied with the e4m3
  operands.

The fused method (the lm_head matmul computed chunk by chunk inside the loss so
the ``(B*T, vocab)`` logits are never materialised -- "Increasing throughput",
fused linear cross-entropy) reaches this same result up to rounding order; the
oracle materialises the logits.  Rows are independent, so large inputs are
processed in blocks of rows; the only cross-row quantities (the loss sum, the
valid count and ``dW``) are plain sums over those blocks.

Targets outside ``[0, Vreal)`` that are not ``ignore_index`` are invalid; they
are counted and treated as ignored (the GPU path raises a status bit for them).

Parity pins (``tests/test_oracle.py``): W = 0 closed form (loss = ln Vreal),
softmax-minus-onehot rows summing to zero, zero gradient in padded rows,
no-softcap case against ``torch.nn.functional.cross_entropy`` in fp64, central
finite differences, and a brute-force per-element loop on tiny shapes.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "logits", "softcap", "softcap_derivative", "valid_rows", "row_forward", "forward",
    "row_dlogits", "backward", "forward_backward", "dW_rows", "rmsnorm_forward",
    "rmsnorm_backward", "rmsnorm_head", "round_bf16", "encode_e5m2", "E5M2_SCALE", "dlogits_e5m2",
    "backward_fp8", "dW_rows_fp8",
]


def logits(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """``z = X W^T``: hidden states [n, d] times the untied LM head [Vpad, d]."""
    return np.asarray(X, np.float64) @ np.asarray(W, np.float64).T


def softcap(z: np.ndarray, cap: float) -> np.ndarray:
    """``s = cap * tanh(z / cap)``; identity when ``cap <= 0``."""
    if cap > 0:
        return cap * np.tanh(z / cap)
    return z


def softcap_derivative(z: np.ndarray, cap: float) -> np.ndarray:
    """``ds/dz = 1 - tanh(z/cap)^2``, evaluated from z (not from s, which would
    cancel badly near saturation); 1 when there is no softcap."""
    if cap > 0:
        th = np.tanh(z / cap)
        return 1.0 - th * th
    return np.ones_like(z)


def valid_rows(t: np.ndarray, Vreal: int, ignore_index: int):
    """Boolean mask of rows that enter the loss, and the number of invalid targets
    (neither ignore_index nor inside [0, Vreal))."""
    t = np.asarray(t, np.int64)
    in_range = (t >= 0) & (t < Vreal)
    ignored = t == ignore_index
    bad = int(np.count_nonzero(~in_range & ~ignored))
    return in_range & ~ignored, bad


def row_forward(X, W, t, Vreal: int, cap: float, ignore_index: int):
    """Per-row log-sum-exp over the real columns and the target's softcapped logit.

    Returns ``(lse [n], s_target [n] (0 for rows not in the loss), valid [n])``."""
    z = logits(X, W)
    s = softcap(z, cap)[:, :Vreal]                       # padded columns excluded
    m = s.max(axis=1)
    lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    valid, _ = valid_rows(t, Vreal, ignore_index)
    rows = np.nonzero(valid)[0]
    s_t = np.zeros(len(t), np.float64)
    s_t[rows] = s[rows, np.asarray(t, np.int64)[rows]]
    return lse, s_t, valid


def forward(X, W, t, Vreal: int, cap: float, ignore_index: int, block_rows: int = 1024):
    """Mean cross entropy over valid rows.  Returns dict(loss, lse [N], n_valid, n_bad)."""
    N = X.shape[0]
    lse = np.empty(N, np.float64)
    total = 0.0
    for r0 in range(0, N, block_rows):
        r1 = min(N, r0 + block_rows)
        l, st, v = row_forward(X[r0:r1], W, t[r0:r1], Vreal, cap, ignore_index)
        lse[r0:r1] = l
        total += float(np.sum((l - st)[v]))
    valid, bad = valid_rows(t, Vreal, ignore_index)
    nv = int(np.count_nonzero(valid))
    loss = total / nv if nv > 0 else 0.0
    return dict(loss=loss, lse=lse, n_valid=nv, n_bad=bad)


def row_dlogits(X, W, t, lse, Vreal: int, cap: float, ignore_index: int, n_valid: int,
                g: float = 1.0, with_parts: bool = False):
    """``dz = g/Nv * (softmax(s) - onehot(t)) * (1 - tanh^2(z/cap))`` for a block of rows.

    Columns ``j >= Vreal`` and rows not in the loss get 0.  With ``with_parts``
    also returns ``g_s = dL/ds`` (softmax minus onehot, scaled) for invariant tests."""
    z = logits(X, W)
    Vpad = z.shape[1]
    s = softcap(z, cap)
    valid, _ = valid_rows(t, Vreal, ignore_index)
    gs = np.zeros_like(z)
    if n_valid > 0:
        p = np.exp(s[:, :Vreal] - np.asarray(lse, np.float64)[:, None])
        rows = np.nonzero(valid)[0]
        p[rows, np.asarray(t, np.int64)[rows]] -= 1.0
        p[~valid] = 0.0
        gs[:, :Vreal] = (g / n_valid) * p
    dz = gs * softcap_derivative(z, cap)
    assert Vpad == W.shape[0]
    return (dz, gs) if with_parts else dz


def backward(X, W, t, Vreal: int, cap: float, ignore_index: int, g: float = 1.0, lse=None,
             block_rows: int = 1024, Xg=None, Wg=None):
    """Gradients of ``g * loss``: ``dX = dz W`` [N, d] and ``dW = dz^T X`` [Vpad, d].

    ``Xg`` / ``Wg`` (default X / W) are the operands of the two gradient products; the logits
    and hence ``dz`` always come from X and W."""
    X = np.asarray(X, np.float64)
    W = np.asarray(W, np.float64)
    Xg = X if Xg is None else np.asarray(Xg, np.float64)
    Wg = W if Wg is None else np.asarray(Wg, np.float64)
    N = X.shape[0]
    valid, _ = valid_rows(t, Vreal, ignore_index)
    nv = int(np.count_nonzero(valid))
    if lse is None:
        lse = forward(X, W, t, Vreal, cap, ignore_index, block_rows)["lse"]
    dX = np.zeros_like(X)
    dW = np.zeros_like(W)
    for r0 in range(0, N, block_rows):
        r1 = min(N, r0 + block_rows)
        dz = row_dlogits(X[r0:r1], W, t[r0:r1], lse[r0:r1], Vreal, cap, ignore_index, nv, g)
        dX[r0:r1] = dz @ Wg
        dW += dz.T @ Xg[r0:r1]
    return dX, dW


def forward_backward(X, W, t, Vreal: int, cap: float, ignore_index: int, g: float = 1.0,
                     block_rows: int = 1024, Xg=None, Wg=None):
    """Loss, lse and both gradients in one call (what one fused training step needs)."""
    f = forward(X, W, t, Vreal, cap, ignore_index, block_rows)
    dX, dW = backward(X, W, t, Vreal, cap, ignore_index, g, f["lse"], block_rows, Xg, Wg)
    f.update(dX=dX, dW=dW)
    return f


def dW_rows(X, W, t, lse, vocab_rows, Vreal: int, cap: float, ignore_index: int,
            g: float = 1.0, block_rows: int = 4096, Xg=None):
    """Selected rows ``j`` of ``dW = dz^T Xg`` (Xg defaults to X), given the lse of every
    token row.

    Only the logit columns ``j`` in ``vocab_rows`` are formed, so this costs
    ``N * d * len(vocab_rows)`` instead of a full backward."""
    X = np.asarray(X, np.float64)
    Xg = X if Xg is None else np.asarray(Xg, np.float64)
    Wj = np.asarray(W, np.float64)[np.asarray(vocab_rows)]
    vocab_rows = np.asarray(vocab_rows, np.int64)
    valid, _ = valid_rows(t, Vreal, ignore_index)
    nv = int(np.count_nonzero(valid))
    out = np.zeros((len(vocab_rows), X.shape[1]), np.float64)
    if nv == 0:
        return out
    t = np.asarray(t, np.int64)
    real = vocab_rows < Vreal
    for r0 in range(0, X.shape[0], block_rows):
        r1 = min(X.shape[0], r0 + block_rows)
        z = X[r0:r1] @ Wj.T                                   # [rows, len(vocab_rows)]
        s = softcap(z, cap)
        p = np.exp(s - np.asarray(lse[r0:r1], np.float64)[:, None])
        p -= (t[r0:r1, None] == vocab_rows[None, :])
        p[~valid[r0:r1]] = 0.0
        p[:, ~real] = 0.0
        dz = (g / nv) * p * softcap_derivative(z, cap)
        out += dz.T @ Xg[r0:r1]
    return out


# ------------------------------------------------------------------------ final RMSNorm
# The model's last RMSNorm feeds the head (the write-ups' model is Llama-style with RMSNorm;
# config appendix: rms_norm_eps = 1.0e-6):  x_i = h_i * rstd_i * gamma,
# rstd_i = 1 / sqrt(mean_k h_ik^2 + eps).

def rmsnorm_forward(H, gamma, eps: float = 1e-6):
    """Returns (x [N, d], rstd [N]) in float64."""
    H = np.asarray(H, np.float64)
    rstd = 1.0 / np.sqrt(np.mean(H * H, axis=1) + eps)
    return H * rstd[:, None] * np.asarray(gamma, np.float64)[None, :], rstd


def rmsnorm_backward(H, gamma, dX, eps: float = 1e-6):
    """Chain rule through x = h * rstd(h) * gamma for an upstream gradient dX = dL/dx.

    Returns (dH [N, d], dgamma [d]):  with xh = h * rstd and g = dX * gamma,
    dH = rstd * (g - xh * mean_k(g * xh)),  dgamma = sum_i dX * xh."""
    H = np.asarray(H, np.float64)
    dX = np.asarray(dX, np.float64)
    gamma = np.asarray(gamma, np.float64)
    rstd = 1.0 / np.sqrt(np.mean(H * H, axis=1) + eps)
    xh = H * rstd[:, None]
    g = dX * gamma[None, :]
    dH = rstd[:, None] * (g - xh * np.mean(g * xh, axis=1, keepdims=True))
    return dH, np.sum(dX * xh, axis=0)


def rmsnorm_head(H, gamma, W, t, Vreal: int, cap: float, ignore_index: int, eps: float = 1e-6,
                 g: float = 1.0, round_x: bool = True, block_rows: int = 1024):
    """The final RMSNorm and the head as one training step: x = rmsnorm(h) -- rounded to bf16
    when ``round_x`` (the head reads the normalised hidden in the model's activation type) --,
    the loss and gradients of the head on x, then the chain rule through the RMSNorm with the
    exact (unrounded) normalised rows.  Returns the ``forward_backward`` dict with ``X`` (the
    head's input), ``dH`` and ``dgamma`` added."""
    x, _ = rmsnorm_forward(H, gamma, eps)
    if round_x:
        x = round_bf16(x)
    f = forward_backward(x, W, t, Vreal, cap, ignore_index, g, block_rows)
    dH, dgamma = rmsnorm_backward(H, gamma, f["dX"], eps)
    f.update(X=x, dH=dH, dgamma=dgamma)
    return f


# ------------------------------------------------------------------------ FP8 gradient products
# The write-ups run all three GEMMs of a linear layer in FP8 with dynamic tensorwise scaling
# ("Increasing throughput": one forward and two backward GEMMs).  Reading adopted for the head
# (the pages give no format for the gradient): the logits operands are e4m3 (as above), the
# softmax gradient is e5m2 -- the format with the wider exponent range, needed because the
# softmax probabilities of one row span many binades -- and the two gradient products multiply
# it with the same e4m3 operands.  The gradient is normalised before it is encoded:
#   dz_ij = g/Nv * dzn_ij,   dzn_ij = (softmax(s_i)_j - [j = t_i]) (1 - tanh^2(z_ij / cap)),
# and |dzn| <= 1, so a fixed power-of-two scale 2^15 (below the e5m2 maximum 57344) covers its
# range without an amax pass; the factor g/(Nv 2^15) and the operands' tensorwise scales are
# applied to the products' fp32 results.  dzn is formed as A_ij / S_i from the unnormalised
# operand A_ij = exp(s_ij - cap)(1 - tanh^2) -- rounded to bf16 -- with S_i = sum_j exp(s_ij -
# cap) and the target element A_{i,t_i} = (1 - tanh^2)(exp(s_{i,t_i} - cap) - S_i), rounded to
# bf16 as well (the reference cap is what keeps exp(s - cap) <= 1 before the row sum is known).

E5M2_SCALE = float(2 ** 15)


def round_bf16(a):
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64."""
    import torch
    return torch.from_numpy(np.asarray(a, np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def encode_e5m2(a):
    """Round float64 values to the nearest e5m2 value (ties to even); |a| <= 57344 here."""
    import torch
    return (torch.from_numpy(np.asarray(a, np.float64)).to(torch.float32)
            .to(torch.float8_e5m2).to(torch.float64).numpy())


def dlogits_e5m2(X, W, t, Vreal: int, cap: float, ignore_index: int, round_operand: bool = True,
                 encode: bool = True):
    """The e5m2 codes (as values, times 2^15) of the normalised softmax gradient dzn of a
    block of rows; rows not in the loss and padded columns are 0.  ``round_operand`` /
    ``encode`` switch the bf16 rounding of A and the e5m2 encoding off (exact dzn * 2^15)."""
    if not cap > 0:
        raise ValueError("the FP8 gradient path takes the reference exp(s - cap): cap > 0")
    z = logits(X, W)
    Vpad = z.shape[1]
    s = softcap(z, cap)
    der = softcap_derivative(z, cap)
    e = np.exp(s - cap)
    e[:, Vreal:] = 0.0
    S = e.sum(axis=1)
    A = e * der
    valid, _ = valid_rows(t, Vreal, ignore_index)
    rows = np.nonzero(valid)[0]
    tt = np.asarray(t, np.int64)[rows]
    A[rows, tt] = der[rows, tt] * (e[rows, tt] - S[rows])
    if round_operand:
        A = round_bf16(A)
    q = A / S[:, None] * E5M2_SCALE
    if encode:
        q = encode_e5m2(q)
    q[~valid] = 0.0
    assert q.shape[1] == Vpad
    return q


def backward_fp8(Xq, Wq, t, Vreal: int, cap: float, ignore_index: int, g: float = 1.0,
                 block_rows: int = 1024, round_operand: bool = True, encode: bool = True):
    """Gradients of ``g * loss`` with FP8 gradient products: dX = g/(Nv 2^15) q Wq and
    dW = g/(Nv 2^15) q^T Xq, q = dlogits_e5m2(...), with Xq / Wq the (dequantised) e4m3
    operands of the logits.  With round_operand = encode = False this is ``backward`` on
    (Xq, Wq)."""
    Xq = np.asarray(Xq, np.float64)
    Wq = np.asarray(Wq, np.float64)
    valid, _ = valid_rows(t, Vreal, ignore_index)
    nv = int(np.count_nonzero(valid))
    dX = np.zeros_like(Xq)
    dW = np.zeros_like(Wq)
    if nv == 0:
        return dX, dW
    f = g / (nv * E5M2_SCALE)
    for r0 in range(0, Xq.shape[0], block_rows):
        r1 = min(Xq.shape[0], r0 + block_rows)
        q = dlogits_e5m2(Xq[r0:r1], Wq, t[r0:r1], Vreal, cap, ignore_index, round_operand,
                         encode)
        dX[r0:r1] = f * (q @ Wq)
        dW += f * (q.T @ Xq[r0:r1])
    return dX, dW


def dW_rows_fp8(Xq, Wq, t, lse, vocab_rows, Vreal: int, cap: float, ignore_index: int,
                g: float = 1.0, block_rows: int = 4096):
    """Selected rows ``j`` of the FP8-path dW (``backward_fp8``), given the lse of every row:
    S_i = exp(lse_i - cap) is the row sum the codes are normalised by, so only the columns in
    ``vocab_rows`` have to be formed."""
    Xq = np.asarray(Xq, np.float64)
    Wj = np.asarray(Wq, np.float64)[np.asarray(vocab_rows)]
    vocab_rows = np.asarray(vocab_rows, np.int64)
    valid, _ = valid_rows(t, Vreal, ignore_index)
    nv = int(np.count_nonzero(valid))
    out = np.zeros((len(vocab_rows), Xq.shape[1]), np.float64)
    if nv == 0:
        return out
    t = np.asarray(t, np.int64)
    real = vocab_rows < Vreal
    for r0 in range(0, Xq.shape[0], block_rows):
        r1 = min(Xq.shape[0], r0 + block_rows)
        z = Xq[r0:r1] @ Wj.T
        s = softcap(z, cap)
        der = softcap_derivative(z, cap)
        e = np.exp(s - cap)
        e[:, ~real] = 0.0
        S = np.exp(np.asarray(lse[r0:r1], np.float64) - cap)
        A = e * der
        hit = t[r0:r1, None] == vocab_rows[None, :]
        A = np.where(hit, der * (e - S[:, None]), A)
        q = encode_e5m2(round_bf16(A) / S[:, None] * E5M2_SCALE)
        q[~valid[r0:r1]] = 0.0
        out += q.T @ Xq[r0:r1]
    return out * (g / (nv * E5M2_SCALE))
