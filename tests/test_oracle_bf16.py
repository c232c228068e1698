"""Oracle pins: the fp32 -> bf16 rounding of dequantize's bf16 output, and the
exact decode of the 1D-column and 2D layouts.

bf16 rounding is pinned to PyTorch's own float32 -> bfloat16 conversion, an
independent implementation of round-to-nearest-even, on random patterns, every
kind of tie, the top of the range (overflow to Inf) and subnormals.  The
decode branches are pinned by exact round trips: a tensor whose blocks hold
grid values with their block maximum at 6 quantizes to scale 2^e with the grid
values as codes ("MXFP4" (aiwiki.ai), "Conversion rules"), and decoding must
return it bit for bit ("Format specification": value = E2M1 * 2^(code-127)).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


def _torch_bf16_bits(f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(f32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _check_against_torch(bits_u32: np.ndarray):
    f = bits_u32.astype(np.uint32).view(np.float32)
    ours = oracle.f32_to_bf16(f)
    ref = _torch_bf16_bits(f)
    nan = np.isnan(f)
    # NaN stays NaN (payloads are not part of the contract)
    assert np.all(np.isnan(synth.bf16_to_f32(ours[nan])))
    bad = np.nonzero(ours[~nan] != ref[~nan])[0]
    assert bad.size == 0, f"first mismatch: f32 bits {bits_u32[~nan][bad[0]]:#010x} -> ours " \
                          f"{ours[~nan][bad[0]]:#06x}, torch {ref[~nan][bad[0]]:#06x}"


def test_bf16_rounding_matches_torch_on_random_patterns():
    g = np.random.default_rng(123)
    _check_against_torch(g.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32))


def test_bf16_rounding_ties_and_neighbours_match_torch():
    g = np.random.default_rng(7)
    hi = g.integers(0, 2**16, size=20_000, dtype=np.uint64).astype(np.uint32) << 16
    # exact ties (low half 0x8000) with both parities of the kept bit, and
    # the patterns one ulp either side of the tie
    pats = np.concatenate([hi | 0x8000, hi | 0x7FFF, hi | 0x8001, hi, hi | 0xFFFF])
    _check_against_torch(pats)


def test_bf16_rounding_range_edges_match_torch():
    edges = []
    for sign in (0, 0x80000000):
        for base in (0x7F7F0000, 0x7F7E0000, 0x00000000, 0x00010000, 0x007F0000, 0x00800000):
            for low in (0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF):
                edges.append(sign | base | low)
        edges += [sign | 0x7F800000, sign | 0x7FC00000, sign | 0x7F800001]   # Inf, NaNs
    # the largest finite fp32 rounds up to Inf; the smallest subnormals round to 0
    _check_against_torch(np.array(edges, np.uint32))


def test_dequantize_bf16_output_is_torch_rounding_of_fp32_output():
    """With the inverse RHT the decoded fp32 values are inexact in bf16; the bf16
    output must be their nearest-even rounding."""
    x = synth.student_t_bf16((64, 64), seed=31)
    for layout in (oracle.LAYOUT_1D_ROW, oracle.LAYOUT_1D_COL, oracle.LAYOUT_2D):
        q = oracle.quantize(x, layout, 32, oracle.ROUND_RNE, seed=8)
        f32, b16 = oracle.dequantize(q[0], q[1], 64, 64, layout, 32, seed=8)
        assert np.array_equal(b16, _torch_bf16_bits(f32))
        assert not np.array_equal(synth.bf16_to_f32(b16), f32)   # the rounding is exercised


def test_round_trip_of_grid_tensor_is_exact_1d_col():
    g = np.random.default_rng(12)
    rows, cols = 96, 96
    vals = g.choice(np.concatenate([GRID, -GRID]), size=(rows, cols))
    vals[::32, :] = -6.0                                  # each column block (32 rows) has amax 6
    exps = g.integers(-100, 100, size=(rows // 32, cols))    # per (row block, column)
    scaled = vals * np.repeat(2.0 ** exps, 32, axis=0)
    x = synth.bf16_bits(scaled.astype(np.float32))
    assert np.array_equal(synth.bf16_to_f32(x).astype(np.float64), scaled)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_COL)
    assert codes.shape == (cols, rows // 2) and scales.shape == (cols, rows // 32)
    assert np.array_equal(scales.astype(int) - 127, exps.T)
    f32, b16 = oracle.dequantize(codes, scales, rows, cols, oracle.LAYOUT_1D_COL)
    assert np.array_equal(f32.astype(np.float64), scaled)
    assert np.array_equal(b16, x)


def test_round_trip_of_grid_tensor_is_exact_2d():
    g = np.random.default_rng(13)
    rows, cols = 96, 128
    vals = g.choice(np.concatenate([GRID, -GRID]), size=(rows, cols))
    vals[::32, ::32] = 6.0                                # each 32x32 tile has amax 6
    exps = g.integers(-100, 100, size=(rows // 32, cols // 32))
    scaled = vals * np.kron(2.0 ** exps, np.ones((32, 32)))
    x = synth.bf16_bits(scaled.astype(np.float32))
    assert np.array_equal(synth.bf16_to_f32(x).astype(np.float64), scaled)
    codes, scales, codes_t = oracle.quantize(x, oracle.LAYOUT_2D, transposed_copy=True)
    assert np.array_equal(scales.astype(int) - 127, exps)
    f32, b16 = oracle.dequantize(codes, scales, rows, cols, oracle.LAYOUT_2D)
    assert np.array_equal(f32.astype(np.float64), scaled)
    assert np.array_equal(b16, x)
    # the transposed copy with the transposed tile scales decodes to x^T
    ft, _ = oracle.dequantize(codes_t, np.ascontiguousarray(scales.T), cols, rows, oracle.LAYOUT_2D)
    assert np.array_equal(ft.astype(np.float64), scaled.T)


@pytest.mark.parametrize("layout", [oracle.LAYOUT_1D_COL, oracle.LAYOUT_2D])
def test_nan_scale_decodes_nan_in_every_layout(layout):
    x = np.full((64, 64), 0x3F80, np.uint16)             # 1.0
    x[5, 7] = 0x7FC0                                     # NaN in the block of (5, 7)
    q = oracle.quantize(x, layout)
    f32, _ = oracle.dequantize(q[0], q[1], 64, 64, layout)
    nan = np.isnan(f32)
    if layout == oracle.LAYOUT_1D_COL:
        expect = np.zeros((64, 64), bool)
        expect[0:32, 7] = True
    else:
        expect = np.zeros((64, 64), bool)
        expect[0:32, 0:32] = True
    assert np.array_equal(nan, expect)
    assert np.all(f32[~nan] == 1.0)
