"""Oracle pins: NVFP4 ("MXFP4" (aiwiki.ai), "Comparison with NVFP4": E2M1
elements, blocks of 16, an FP8 E4M3 block scale fitted to each block, a
per-tensor FP32 scale, 4.5 bits per value).  The scale rule itself is the
oracle's reading R16; what pins it here is what the page and the formats fix.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def test_storage_is_4_5_bits_per_value():
    bits = 16 * 4 + 8                     # 16 E2M1 codes + one E4M3 scale
    assert bits / 16 == 4.5
    assert (32 * 4 + 8) / 32 == 4.25      # MXFP4, for the page's comparison


def test_e4m3_decode_matches_torch_float8():
    """Every E4M3 byte decodes as PyTorch's float8_e4m3fn does (NaN at 0x7F, 0xFF)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.nanmax(got) == 448.0


def test_e4m3_rounding_matches_torch_below_max():
    """Nearest-even E4M3 of non-negative values up to 448 equals PyTorch's
    float32 -> float8_e4m3fn conversion (ties included: midpoints of adjacent
    codes are tried explicitly); above 448 the oracle saturates at 448."""
    vals = [oracle.e4m3_decode(c) for c in range(0x7F)]
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    rng = np.random.default_rng(3)
    xs = np.concatenate([vals, mids, rng.uniform(0, 448, 4000), np.exp(rng.uniform(-12, 6, 2000))])
    xs = xs[xs <= 448].astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rne(float(v)) for v in xs], np.uint8)
    assert np.array_equal(got, ref)
    assert oracle.e4m3_rne(500.0) == 0x7E and oracle.e4m3_rne(1e9) == 0x7E


def test_largest_block_scale_is_e4m3_max():
    """With S = amax / (6 * 448) the block holding the tensor maximum gets the
    largest E4M3 scale, 448, and that maximum is stored as 6."""
    x = synth.student_t_bf16((64, 256), seed=31)
    codes, scales, amax = oracle.nvfp4_quantize(x, oracle.LAYOUT_1D_ROW)
    v = np.abs(synth.bf16_to_f32(x))
    r, c = np.unravel_index(np.argmax(v), v.shape)
    assert oracle.e4m3_decode(int(scales[r, c // 16])) == 448.0
    nib = (int(codes[r, c // 2]) >> (4 * (c % 2))) & 7
    assert nib == 7                                               # 6
    assert amax == float(v.max())


def test_e4m3_scale_fits_block_maxima_closer_than_e8m0():
    """The page's point: an E8M0 scale snaps to a power of two and can leave a
    large error on the block maximum; an E4M3 scale fits each block more
    closely.  Mean relative error of the dequantized block maxima."""
    x = synth.normal_bf16((256, 512), 32)
    v = synth.bf16_to_f32(x).astype(np.float64)
    nc, ns, amax = oracle.nvfp4_quantize(x, oracle.LAYOUT_1D_ROW)
    nv = oracle.nvfp4_dequantize(nc, ns, 256, 512, oracle.LAYOUT_1D_ROW, amax).astype(np.float64)
    mc, ms = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    mxv, _ = oracle.dequantize(mc, ms, 256, 512, oracle.LAYOUT_1D_ROW)
    def block_max_err(deq, bs):
        vb, db = v.reshape(-1, bs), deq.astype(np.float64).reshape(-1, bs)
        i = np.argmax(np.abs(vb), axis=1)
        t = np.abs(vb[np.arange(len(i)), i])
        return np.mean(np.abs(np.abs(db[np.arange(len(i)), i]) - t) / t)
    assert block_max_err(nv, 16) < 0.5 * block_max_err(mxv, 32)


def test_dequantize_within_half_a_grid_step():
    """Unsaturated elements dequantize within half an E2M1 step times the block divisor."""
    x = synth.student_t_bf16((128, 128), seed=33)
    codes, scales, amax = oracle.nvfp4_quantize(x, oracle.LAYOUT_1D_ROW)
    deq = oracle.nvfp4_dequantize(codes, scales, 128, 128, oracle.LAYOUT_1D_ROW, amax).astype(np.float64)
    v = synth.bf16_to_f32(x).astype(np.float64)
    S = oracle.nvfp4_tensor_scale(amax)
    X = np.repeat(np.array([[oracle.e4m3_decode(int(s)) for s in row] for row in scales]) * S, 16, axis=1)
    ok = np.abs(v) <= 6 * X
    step = np.where(np.abs(v) < 2 * X, 0.5, np.where(np.abs(v) < 4 * X, 1.0, 2.0)) * X
    assert np.all(np.abs(v - deq)[ok] <= 0.5 * step[ok] * (1 + 1e-6))


def test_column_layout_is_row_layout_of_transpose():
    x = synth.student_t_bf16((96, 64), seed=34)
    cc, sc, ac = oracle.nvfp4_quantize(x, oracle.LAYOUT_1D_COL, oracle.ROUND_SR, 7)
    cr, sr_, ar = oracle.nvfp4_quantize(np.ascontiguousarray(x.T), oracle.LAYOUT_1D_ROW, oracle.ROUND_SR, 7)
    assert np.array_equal(cc, cr) and np.array_equal(sc, sr_) and ac == ar


def test_special_tensors():
    z = np.zeros((32, 32), np.uint16)
    c, s, a = oracle.nvfp4_quantize(z, oracle.LAYOUT_1D_ROW)
    assert a == 0.0 and not c.any() and not s.any()
    x = synth.normal_bf16((32, 32), 5)
    x[3, 7] = 0x7FC0                                              # NaN
    c, s, a = oracle.nvfp4_quantize(x, oracle.LAYOUT_1D_ROW)
    assert math.isnan(a) and np.all(s == 0x7F) and not c.any()


def test_gemm_equals_matmul_of_dequantized_operands():
    """C = S_a S_b sum over 16-blocks s_a s_b sum a b, which is the product of
    the exactly dequantized operands (every term is exact in fp64)."""
    a = synth.normal_bf16((48, 96), 35)
    b = synth.normal_bf16((40, 96), 36)
    ca, sa, aa = oracle.nvfp4_quantize(a, oracle.LAYOUT_1D_ROW)
    cb, sb, ab = oracle.nvfp4_quantize(b, oracle.LAYOUT_1D_ROW)
    def deq64(c, s, amax, rows, k):
        S = float(np.float32(amax) / np.float32(2688.0))
        vals = np.zeros((rows, k))
        for r in range(rows):
            for j in range(k):
                nib = (int(c[r, j // 2]) >> (4 * (j % 2))) & 0xF
                vals[r, j] = oracle.e2m1_decode(nib) * oracle.e4m3_decode(int(s[r, j // 16])) * S
        return vals
    ref = deq64(ca, sa, aa, 48, 96) @ deq64(cb, sb, ab, 40, 96).T
    pairs = [(m, n) for m in range(48) for n in range(40)]
    got, _ = oracle.nvfp4_gemm_entries(ca, sa, aa, cb, sb, ab, 96, pairs)
    assert np.allclose(got.reshape(48, 40), ref, rtol=1e-12, atol=0)
