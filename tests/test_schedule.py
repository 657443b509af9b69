"""Host-side checks of the persistent tile schedule of the contraction kernels (no GPU).

The assignment function is the kernels' own (compiled for the host too and exposed as
flce_check_pair_schedule): every tile of both problems must go to exactly one (pair, slot),
and on the workloads the bench runs the per-pair work must be balanced.
"""
import numpy as np
import pytest

from lm_head_linear_gemm_b200 import _abi

PAIRS = 74          # SM pairs of a 148-SM B200


def kblocks(K):     # 64 bf16 per k-block
    return (K + 63) // 64


def tiles(M, N, bm=256, bn=256):
    return ((M + bm - 1) // bm) * ((N + bn - 1) // bn)


@pytest.mark.parametrize("rows,d", [(4096, 3072), (8192, 3072), (16384, 3072), (4096, 1536),
                                    (2048, 3072), (1024, 3072), (300, 200)])
def test_gradient_launch_is_balanced(rows, d):
    """dX (wide 256 x 512 tiles when d has an even number of 256-blocks) next to dW."""
    Vpad = 50304
    nb = (d + 255) // 256
    wide = nb % 2 == 0
    T0 = tiles(rows, d, bn=512 if wide else 256)
    c0 = kblocks(Vpad) * (2 if wide else 1)
    T1, c1 = tiles(Vpad, d), kblocks(rows)
    hi, lo = _abi.check_pair_schedule(PAIRS, T0, c0, T1, c1)
    total = T0 * c0 + T1 * c1
    assert hi * PAIRS >= total >= lo * PAIRS
    if rows >= 2048:                      # enough short tiles to even out the long ones
        assert (hi - lo) / hi <= 0.05, (hi, lo)
        # the busiest pair within two short tiles of the mean
        assert hi - total / PAIRS < 2 * c1, (hi, total / PAIRS, c1)


def test_logits_launch_round_robin():
    T0, c0 = tiles(4096, 50304), kblocks(3072)
    hi, lo = _abi.check_pair_schedule(PAIRS, T0, c0, 0, 1)
    assert hi - lo == c0          # 3152 tiles on 74 pairs: 42 or 43 each


def test_random_shapes_cover_every_tile_once():
    rng = np.random.default_rng(7)
    for _ in range(3000):
        pairs = int(rng.integers(1, 100))
        T0 = int(rng.integers(0, 400))
        T1 = int(rng.integers(0, 3000))
        c0 = int(rng.integers(1, 2000))
        c1 = int(rng.integers(1, 200))
        _abi.check_pair_schedule(pairs, T0, c0, T1, c1)


def test_fewer_tiles_than_pairs():
    for T0, T1 in ((1, 0), (3, 5), (0, 7), (73, 1), (75, 0)):
        _abi.check_pair_schedule(PAIRS, T0, 100, T1, 10)


@pytest.mark.parametrize("args", [(0, 1, 1, 1, 1), (5000, 1, 1, 1, 1), (4, -1, 1, 1, 1),
                                  (4, 1, 0, 1, 1), (4, 1, 1, 1, 0), (4, 1 << 25, 1, 0, 1)])
def test_rejects_bad_sizes(args):
    with pytest.raises(_abi.FlceError):
        _abi.check_pair_schedule(*args)
