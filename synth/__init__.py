"""Seeded synthetic inputs for the fused LM-head linear + softcapped cross-entropy.

This module is shared by the fp64 oracle (``oracle/``), the tests and ``bench.py``.
It draws random numbers and rounds them to bf16; it holds none of the loss's
arithmetic (no matmul, softcap, softmax or gradient).

Workload shapes follow the little-lm 3.8B write-ups: the untied LM head is
``[50304, 3072]`` (154.5M parameters, "Setup" table of the write-up and the
config appendix), the GPT-2 vocabulary of 50257 tokens is padded to 50304, a
multiple of 64 (config appendix, "Increasing throughput"), and the logit softcap
is 15.0 (the config appendix sets it for the model and for its fused loss).  The pages train on
ClimbMix text through the GPT-2 tokenizer; that data is not available, so
targets are drawn from a truncated Zipf law over the real vocabulary as a
stand-in for natural-text token frequencies.

bf16 tensors are returned as ``numpy.uint16`` bit patterns; ``bf16_to_f64`` and
``bf16_to_f32`` widen them exactly.
"""
from __future__ import annotations

import dataclasses
import zlib

import numpy as np

__all__ = [
    "FlceConfig", "CONFIGS", "make_inputs", "make_fp8_inputs", "quantize_e4m3", "e4m3_to_f64",
    "f32_to_bf16_bits", "bf16_to_f32", "bf16_to_f64", "zipf_targets", "uniform_targets",
    "place_ignored",
]


@dataclasses.dataclass(frozen=True)
class FlceConfig:
    """One synthetic workload of the fused linear cross-entropy."""
    name: str
    N: int                 # tokens (rows of X)
    d: int                 # hidden size
    Vreal: int             # real vocabulary
    Vpad: int              # padded vocabulary (rows of W)
    x_dist: str            # "normal": N(0,1) per element; "unit_rms": rows scaled to RMS 1
    w_std: float           # W ~ N(0, w_std^2), all Vpad rows (padded rows are real rows)
    target_dist: str       # "uniform" or "zipf"
    ignore_count: int      # how many positions carry ignore_index
    ignore_index: int = -1
    cap: float = 15.0
    seed: int = 0
    zipf_s: float = 1.1


def _ignored(frac: float, n: int) -> int:
    return int(round(frac * n))


CONFIGS = {
    # N=64, d=128, V 1000 -> 1024; two ignored positions.
    "tiny": FlceConfig("tiny", 64, 128, 1000, 1024, "normal", 0.02, "uniform", 2),
    # batch 8 x ctx 1024, d=1536.
    "small": FlceConfig("small", 8192, 1536, 50257, 50304, "unit_rms", 0.02, "zipf",
                        _ignored(0.02, 8192)),
    # the 3.8B model's head: batch 16 x ctx 1024, d=3072.
    "3.8b": FlceConfig("3.8b", 16384, 3072, 50257, 50304, "unit_rms", 0.02, "zipf",
                       _ignored(0.02, 16384)),
    # 3.8B head at 2048 context; wider W so more logits reach the softcap's curved range.
    "3.8b-2k": FlceConfig("3.8b-2k", 32768, 3072, 50257, 50304, "unit_rms", 0.05, "zipf",
                          _ignored(0.02, 32768)),
    # large micro-batch, X and W also given as e4m3 with tensorwise scales (make_fp8_inputs)
    "fp8": FlceConfig("fp8", 65536, 3072, 50257, 50304, "unit_rms", 0.02, "zipf",
                      _ignored(0.05, 65536)),
}

E4M3_MAX = 448.0   # largest finite e4m3 value


def quantize_e4m3(bits_bf16: np.ndarray):
    """Tensorwise e4m3 encoding of bf16 values: scale = amax/448 (fp32), codes =
    e4m3(x / scale) with the fp32 quotient rounded to nearest even by torch's float8_e4m3fn
    cast.  Returns (uint8 codes, float32 scale)."""
    import torch
    x = bf16_to_f32(bits_bf16)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    scale = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
    q = torch.from_numpy(np.ascontiguousarray(x / scale, dtype=np.float32))
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Exact value of e4m3 codes (finite codes only)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def make_fp8_inputs(cfg: FlceConfig | str = "fp8", seed: int | None = None, N: int | None = None):
    """make_inputs plus e4m3 codes and tensorwise scales of X and W (the bf16 arrays stay as
    the reference copies)."""
    inp = make_inputs(cfg, seed=seed, N=N)
    inp["X8"], inp["sX"] = quantize_e4m3(inp["X"])
    inp["W8"], inp["sW"] = quantize_e4m3(inp["W"])
    return inp


def _rng(seed: int, tag: str) -> np.random.Generator:
    """Independent stream per (seed, tensor tag); PCG64 seeded from both."""
    return np.random.Generator(np.random.PCG64([seed, zlib.crc32(tag.encode())]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); returns uint16 bits.

    Inputs here are finite normals, so no NaN handling is needed."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_to_f32(b).astype(np.float64)


def _normal_bf16(rng: np.random.Generator, shape, std: float, chunk_rows: int = 4096):
    rows, cols = shape
    out = np.empty(shape, dtype=np.uint16)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        a = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        out[r0:r1] = f32_to_bf16_bits(a)
    return out


def _unit_rms_bf16(rng: np.random.Generator, shape, chunk_rows: int = 4096):
    """Rows of N(0,1) scaled in fp64 to root-mean-square 1, then rounded to bf16
    (the hidden state after a final RMSNorm with unit gain)."""
    rows, cols = shape
    out = np.empty(shape, dtype=np.uint16)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        a = rng.standard_normal((r1 - r0, cols), dtype=np.float32).astype(np.float64)
        a /= np.sqrt(np.mean(a * a, axis=1, keepdims=True))
        out[r0:r1] = f32_to_bf16_bits(a.astype(np.float32))
    return out


def uniform_targets(rng: np.random.Generator, n: int, vreal: int) -> np.ndarray:
    return rng.integers(0, vreal, size=n, dtype=np.int64)


def zipf_targets(rng: np.random.Generator, n: int, vreal: int, s: float) -> np.ndarray:
    """Truncated Zipf over ranks 1..vreal, P(k) proportional to k^-s, by inverse CDF;
    token id = rank - 1, so id 0 is the most frequent."""
    w = np.arange(1, vreal + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vreal - 1).astype(np.int64)


def place_ignored(rng: np.random.Generator, t: np.ndarray, count: int, ignore_index: int):
    """Set exactly ``count`` seeded positions (a permutation prefix) to ignore_index."""
    if count > 0:
        pos = rng.permutation(t.shape[0])[:count]
        t[pos] = ignore_index
    return t


def make_inputs(cfg: FlceConfig | str, seed: int | None = None, N: int | None = None):
    """Return dict(X=uint16 [N,d] bf16 bits, W=uint16 [Vpad,d], targets=int64 [N], cfg=...).

    ``N`` overrides the row count (the ignored count scales with it)."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    if N is not None and N != cfg.N:
        frac = cfg.ignore_count / cfg.N
        cfg = dataclasses.replace(cfg, N=N, ignore_count=_ignored(frac, N) if cfg.name != "tiny"
                                  else min(cfg.ignore_count, N))
    if seed is not None:
        cfg = dataclasses.replace(cfg, seed=seed)
    s = cfg.seed
    if cfg.x_dist == "normal":
        X = _normal_bf16(_rng(s, "X"), (cfg.N, cfg.d), 1.0)
    elif cfg.x_dist == "unit_rms":
        X = _unit_rms_bf16(_rng(s, "X"), (cfg.N, cfg.d))
    else:
        raise ValueError(cfg.x_dist)
    W = _normal_bf16(_rng(s, "W"), (cfg.Vpad, cfg.d), cfg.w_std)
    rt = _rng(s, "targets")
    if cfg.target_dist == "uniform":
        t = uniform_targets(rt, cfg.N, cfg.Vreal)
    elif cfg.target_dist == "zipf":
        t = zipf_targets(rt, cfg.N, cfg.Vreal, cfg.zipf_s)
    else:
        raise ValueError(cfg.target_dist)
    place_ignored(_rng(s, "ignore"), t, cfg.ignore_count, cfg.ignore_index)
    return dict(X=X, W=W, targets=t, cfg=cfg)


def make_rmsnorm_inputs(cfg: FlceConfig | str, seed: int | None = None, N: int | None = None,
                        h_std: float = 2.0, gamma_std: float = 0.1):
    """make_inputs plus the rows before the model's final RMSNorm and its gain:
    H = uint16 [N,d] bf16 bits of N(0, h_std) (the residual stream has no fixed scale),
    gamma = uint16 [d] bf16 bits of 1 + N(0, gamma_std)."""
    inp = make_inputs(cfg, seed, N)
    c = inp["cfg"]
    inp["H"] = _normal_bf16(_rng(c.seed, "H"), (c.N, c.d), h_std)
    g = 1.0 + gamma_std * _rng(c.seed, "gamma").standard_normal(c.d, dtype=np.float32)
    inp["gamma"] = f32_to_bf16_bits(g.astype(np.float32))
    return inp


def custom_config(name: str, N: int, d: int, Vreal: int, Vpad: int, *, x_dist="normal",
                  w_std=0.02, target_dist="uniform", ignore_count=0, ignore_index=-1,
                  cap=15.0, seed=0) -> FlceConfig:
    """A config outside the named set (parity sizes, edge cases)."""
    return FlceConfig(name, N, d, Vreal, Vpad, x_dist, w_std, target_dist, ignore_count,
                      ignore_index, cap, seed)
