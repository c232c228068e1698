"""Oracle pins: tensor-level quantization and dequantization.

Invariants that follow from the definitions on "MXFP4" (aiwiki.ai):
1D-column blocks are 1D-row blocks of the transpose; a 2D block's scale is the
largest of its row-block scales (floor(log2) is monotone); every element code
is the scalar conversion of the scaled value; the transposed copy is a
permutation; decoding a quantized grid tensor gives it back exactly (this pins
the nibble order and the decode table together); NaN/Inf/zero blocks follow
readings R3/R4; sharded SR with element offsets equals the whole.
"""
import math

import numpy as np
import pytest

import oracle
import synth

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


def nibbles(codes, n):
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)[:, :n]


def decode(codes, n):
    nib = nibbles(codes, n)
    mag = GRID[nib & 7]
    return np.where(nib & 8, -mag, mag)


@pytest.mark.parametrize("rht", [0, 16, 32])
@pytest.mark.parametrize("rnd", [oracle.ROUND_RNE, oracle.ROUND_SR])
def test_col_layout_is_row_layout_of_transpose(rht, rnd):
    x = synth.student_t_bf16((96, 64), seed=3)
    c_col, s_col = oracle.quantize(x, oracle.LAYOUT_1D_COL, rht, rnd, seed=5)
    c_row, s_row = oracle.quantize(np.ascontiguousarray(x.T), oracle.LAYOUT_1D_ROW, rht, rnd, seed=5)
    assert np.array_equal(c_col, c_row) and np.array_equal(s_col, s_row)


@pytest.mark.parametrize("rht", [0, 32])
def test_2d_scale_is_max_of_row_scales_and_codes_are_scalar_conversions(rht):
    x = synth.student_t_bf16((64, 96), seed=4)
    c2, s2, ct = oracle.quantize(x, oracle.LAYOUT_2D, rht, oracle.ROUND_RNE, seed=9, transposed_copy=True)
    _, s1 = oracle.quantize(x, oracle.LAYOUT_1D_ROW, rht, oracle.ROUND_RNE, seed=9)
    for br in range(2):
        for bc in range(3):
            assert s2[br, bc] == s1[br * 32:(br + 1) * 32, bc].max()
    # element codes = scalar RNE of y / X with the 2D scale
    y = synth.bf16_to_f32(x).copy()
    if rht:
        mask = oracle.rht_sign_mask(9)
        for r in range(64):
            for s in range(0, 96, 32):
                y[r, s:s + 32] = oracle.rht_forward(y[r, s:s + 32], mask)
    nib = nibbles(c2, 96)
    for r in range(0, 64, 7):
        for c in range(0, 96, 5):
            e = int(s2[r // 32, c // 32]) - 127
            v = float(np.ldexp(np.float32(y[r, c]), -e).astype(np.float32))
            assert nib[r, c] == oracle.e2m1_rne(v)
    # the transposed copy is a permutation of the same codes
    assert np.array_equal(nibbles(ct, 64), nib.T)


def test_round_trip_of_grid_tensor_is_exact():
    g = np.random.default_rng(11)
    rows, cols = 64, 128
    vals = g.choice(np.concatenate([GRID, -GRID]), size=(rows, cols))
    vals[:, ::32] = 6.0                              # block amax 6 -> X = 1
    exps = g.integers(-100, 100, size=(rows, cols // 32))
    scaled = vals * np.repeat(2.0 ** exps, 32, axis=1)
    x = synth.bf16_bits(scaled.astype(np.float32))
    assert np.array_equal(synth.bf16_to_f32(x).astype(np.float64), scaled)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    assert np.array_equal(scales.astype(int) - 127, exps)
    assert np.array_equal(decode(codes, cols), vals)
    f32, b16 = oracle.dequantize(codes, scales, rows, cols, oracle.LAYOUT_1D_ROW)
    assert np.array_equal(f32.astype(np.float64), scaled)
    assert np.array_equal(b16, x)


def test_packing_order_low_nibble_first():
    vals = np.zeros((1, 32), np.float32)
    vals[0, 0] = 6.0   # code 7 in the low nibble of byte 0
    vals[0, 1] = 0.5   # code 1 in the high nibble of byte 0
    vals[0, 3] = -1.0  # code 0xA in the high nibble of byte 1
    codes, scales = oracle.quantize(synth.bf16_bits(vals), oracle.LAYOUT_1D_ROW)
    assert scales[0, 0] == 127
    assert codes[0, 0] == 0x17 and codes[0, 1] == 0xA0


def test_nan_inf_zero_blocks():
    vals = np.ones((4, 64), np.float32)
    vals[0, 3] = np.nan
    vals[1, 40] = np.inf
    vals[2, :32] = 0.0
    vals[3, :32] = -0.0
    x = synth.bf16_bits(vals)
    x[0, 3] = 0x7FC0                                 # quiet NaN bit pattern
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    assert scales[0, 0] == 0xFF and np.all(codes[0, :16] == 0) and scales[0, 1] == 125
    assert scales[1, 1] == 0xFF and np.all(codes[1, 16:] == 0) and scales[1, 0] == 125
    assert scales[2, 0] == 0 and np.all(codes[2, :16] == 0)
    assert scales[3, 0] == 0 and np.all(codes[3, :16] == 0x88)   # reading R7: -0 kept
    f32, _ = oracle.dequantize(codes, scales, 4, 64, oracle.LAYOUT_1D_ROW)
    assert np.all(np.isnan(f32[0, :32])) and np.all(f32[0, 32:] == 1.0)
    assert np.all(np.isnan(f32[1, 32:]))
    assert np.all(f32[2, :32] == 0)


@pytest.mark.parametrize("layout", [oracle.LAYOUT_1D_ROW, oracle.LAYOUT_1D_COL, oracle.LAYOUT_2D])
def test_sharded_sr_with_offsets_equals_whole(layout):
    x = synth.student_t_bf16((128, 64), seed=21)
    whole = oracle.quantize(x, layout, 32, oracle.ROUND_SR, seed=42)
    if layout == oracle.LAYOUT_1D_COL:
        # shard the output rows (= input columns); offset = output row * output cols
        a = oracle.quantize(np.ascontiguousarray(x[:, :32]), layout, 32, oracle.ROUND_SR, 42, 0)
        b = oracle.quantize(np.ascontiguousarray(x[:, 32:]), layout, 32, oracle.ROUND_SR, 42, 32 * 128)
    else:
        a = oracle.quantize(np.ascontiguousarray(x[:64]), layout, 32, oracle.ROUND_SR, 42, 0)
        b = oracle.quantize(np.ascontiguousarray(x[64:]), layout, 32, oracle.ROUND_SR, 42, 64 * 64)
    for w, pa, pb in zip(whole, a, b):
        assert np.array_equal(w, np.concatenate([pa, pb], axis=0))


@pytest.mark.parametrize("rnd", [oracle.ROUND_RNE, oracle.ROUND_SR])
def test_token_slices_of_column_layout_equal_the_whole(rnd):
    """A slice of tokens (rows of x) quantized along tokens is a column range of
    the whole tensor's output view: with the whole view's row length (sr_ld =
    total tokens) and the slice's first token as offset, every slice draws the
    whole tensor's SR words (reading R8), so the slices' codes and scales are the
    whole's, bit for bit.  Row blocks of the same slice need only the offset."""
    x = synth.student_t_bf16((256, 96), seed=23)
    whole_c, whole_s = oracle.quantize(x, oracle.LAYOUT_1D_COL, 32, rnd, seed=42)
    whole_rc, whole_rs = oracle.quantize(x, oracle.LAYOUT_1D_ROW, 0, rnd, seed=42)
    for t0, n in ((0, 64), (64, 128), (192, 64)):
        part = np.ascontiguousarray(x[t0:t0 + n])
        c, s = oracle.quantize(part, oracle.LAYOUT_1D_COL, 32, rnd, seed=42, elem_offset=t0, sr_ld=256)
        assert np.array_equal(c, whole_c[:, t0 // 2:(t0 + n) // 2])
        assert np.array_equal(s, whole_s[:, t0 // 32:(t0 + n) // 32])
        rc, rs = oracle.quantize(part, oracle.LAYOUT_1D_ROW, 0, rnd, seed=42, elem_offset=t0 * 96)
        assert np.array_equal(rc, whole_rc[t0:t0 + n]) and np.array_equal(rs, whole_rs[t0:t0 + n])
    if rnd == oracle.ROUND_SR:
        # without the whole view's row length the slice draws other words
        c, _ = oracle.quantize(np.ascontiguousarray(x[64:192]), oracle.LAYOUT_1D_COL, 32, rnd, seed=42,
                               elem_offset=64)
        assert not np.array_equal(c, whole_c[:, 32:96])


@pytest.mark.parametrize("rht", [16, 32])
def test_dequantize_inverts_rht(rht):
    x = synth.normal_bf16((32, 64), 5)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW, rht, oracle.ROUND_RNE, seed=3)
    plain, _ = oracle.dequantize(codes, scales, 32, 64, oracle.LAYOUT_1D_ROW)
    back, _ = oracle.dequantize(codes, scales, 32, 64, oracle.LAYOUT_1D_ROW, rht, seed=3)
    mask = oracle.rht_sign_mask(3)
    for r in range(32):
        for s in range(0, 64, rht):
            assert np.array_equal(back[r, s:s + rht], oracle.rht_inverse(plain[r, s:s + rht], mask))
    # the quantization error after the round trip is of the order of the FP4 step
    xf = synth.bf16_to_f32(x)
    err = np.abs(back - xf)
    assert np.median(err) < 0.25 * np.median(np.abs(xf)) + 1e-3


def test_clipping_fraction_is_a_few_percent():
    """Soft check of the ~3% clipping remark (page section "Clipping in the
    reference algorithm"); distribution dependent, so only a loose range."""
    x = synth.normal_bf16((256, 1024), 13)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    y = synth.bf16_to_f32(x).astype(np.float64)
    X = np.repeat(2.0 ** (scales.astype(int) - 127), 32, axis=1)
    frac = float(np.mean(np.abs(y / X) > 6.0))
    assert 0.0 < frac < 0.1
