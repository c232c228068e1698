"""Oracle pins: stochastic rounding.

"MXFP4" (aiwiki.ai), "Training with MXFP4": stochastic rounding gives unbiased
gradients.  Reading R8 fixes the rule (round up iff r < f * 2^32 on a Philox
word).  Pins: unbiasedness within a stated statistical bound over 2^22
element indices, results confined to the two neighbouring grid values, grid
values never move, and the deterministic count of round-ups.
"""
import numpy as np
import pytest

import oracle
import synth

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


def _decode_codes(codes, n):
    lo = codes & 0xF
    hi = codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)[:, :n]
    mag = GRID[nib & 7]
    return np.where(nib & 8, -mag, mag)


# values exactly representable in bf16, away from the grid
VALUES = [0.30078125, 0.8984375, 1.2265625, 1.9921875, 2.703125, 3.3125, 4.5, 5.875, 0.015625]


@pytest.mark.parametrize("v", VALUES)
def test_sr_is_unbiased(v):
    n_blocks = (1 << 22) // 31 + 1
    vals = np.full((n_blocks, 32), v, np.float32)
    vals[:, 0] = 4.0                                   # block amax 4 -> X = 1 exactly
    sign = np.where(np.arange(n_blocks) % 2 == 0, 1.0, -1.0).astype(np.float32)
    vals[:, 1:] *= sign[:, None]
    x = synth.bf16_bits(vals)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW, rnd=oracle.ROUND_SR, seed=1234)
    assert np.all(scales == 127)
    dec = _decode_codes(codes, 32)[:, 1:] * sign[:, None]
    N = dec.size
    lo = GRID[GRID <= v].max()
    hi = GRID[GRID > v].min()
    assert set(np.unique(dec)) <= {lo, hi}
    # the mean of N Bernoulli-mixture draws has sd <= (hi - lo) / (2 sqrt(N))
    bound = 6 * (hi - lo) / (2 * np.sqrt(N))
    assert abs(dec.mean() - v) <= bound, (dec.mean(), v, bound)


def test_sr_round_up_count_is_the_philox_threshold_count():
    v = 1.2265625                                      # lo = 1, hi = 1.5, f = 0.453125
    f = (v - 1.0) / 0.5
    n_blocks = 4096
    vals = np.full((n_blocks, 32), v, np.float32)
    vals[:, 0] = 4.0
    x = synth.bf16_bits(vals)
    seed = 77
    codes, _ = oracle.quantize(x, oracle.LAYOUT_1D_ROW, rnd=oracle.ROUND_SR, seed=seed)
    dec = _decode_codes(codes, 32)
    words = oracle.sr_words(seed, 0, n_blocks * 32).reshape(n_blocks, 32)
    expect_up = words[:, 1:].astype(np.float64) < f * 2.0 ** 32
    assert np.array_equal(dec[:, 1:] == 1.5, expect_up)


def test_sr_leaves_grid_values_and_saturates():
    for g in GRID:
        for r in (0, 1, 2 ** 31, 2 ** 32 - 1):
            assert abs(oracle.e2m1_decode(oracle.e2m1_sr(float(g), r))) == g
            assert abs(oracle.e2m1_decode(oracle.e2m1_sr(float(-g), r))) == g
    for big in (6.5, 7.9, 100.0):
        assert oracle.e2m1_sr(big, 0) == 7 and oracle.e2m1_sr(-big, 0) == 15


def test_sr_extreme_words():
    # r = 0 rounds up any value strictly above lo; r = 2^32 - 1 never rounds up
    # unless f * 2^32 exceeds it (f < 1 here), so it always rounds down.
    for v in (0.3, 1.1, 2.2, 4.4, 5.99):
        lo = GRID[GRID <= v].max()
        hi = GRID[GRID > v].min()
        assert abs(oracle.e2m1_decode(oracle.e2m1_sr(v, 0))) == hi
        assert abs(oracle.e2m1_decode(oracle.e2m1_sr(v, 2 ** 32 - 1))) == lo
