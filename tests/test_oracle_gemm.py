"""Oracle pins: block-scaled dot products and GEMM.

"MXFP4" (aiwiki.ai), "Conversion rules": C = X(A) X(B) sum_i Pi(A) Pi(B) per
block, blocks summed, FP32 result.  The oracle computes it exactly in fp64.
Pins: a hand-worked block pair, agreement with numpy's fp64 matmul of the
decoded operands (a library routine), NaN propagation, and the 2D scale modes
against per-row expanded scales.
"""
import numpy as np
import pytest

import oracle
import synth


def test_single_block_pair_by_hand():
    # A block: first elements 6, -1.5, rest 0.5; scale 2^3.  B block: 2, 4, rest -0.5; scale 2^-2.
    a = np.full((1, 32), 0.5, np.float32)
    a[0, 0], a[0, 1] = 6.0, -1.5
    b = np.full((1, 32), -0.5, np.float32)
    b[0, 0], b[0, 1] = 2.0, 4.0
    a *= 8.0
    b *= 0.25
    ca, sa = oracle.quantize(synth.bf16_bits(a), oracle.LAYOUT_1D_ROW)
    cb, sb = oracle.quantize(synth.bf16_bits(b), oracle.LAYOUT_1D_ROW)
    assert sa[0, 0] == 127 + 3 and sb[0, 0] == 127 - 2
    c, s = oracle.gemm(ca, sa, cb, sb, 32)
    inner = 6 * 2 + (-1.5) * 4 + 30 * (0.5 * -0.5)     # = -1.5
    assert c[0, 0] == 2.0 ** 3 * 2.0 ** -2 * inner
    assert s[0, 0] == 2.0 ** 1 * (12 + 6 + 30 * 0.25)


def _decode_tensor(codes, scales, K, mode=0):
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    lo, hi = codes & 0xF, codes >> 4
    nib = np.stack([lo, hi], -1).reshape(codes.shape[0], -1)[:, :K]
    mag = grid[nib & 7]
    val = np.where(nib & 8, -mag, mag)
    rows = codes.shape[0]
    if mode == 0:
        sc = scales[:, :K // 32]
    elif mode == 1:
        sc = np.repeat(scales, 32, axis=0)[:rows, :K // 32]
    else:
        sc = np.repeat(scales.T, 32, axis=0)[:rows, :K // 32]
    X = np.where(sc == 255, np.nan, 2.0 ** (sc.astype(np.float64) - 127))
    return val * np.repeat(X, 32, axis=1)


@pytest.mark.parametrize("M,N,K", [(16, 24, 64), (33, 7, 256), (64, 96, 2880 // 10)])
def test_gemm_matches_numpy_matmul_of_decoded_operands(M, N, K):
    K = K // 32 * 32
    a = synth.normal_bf16((M, K), 1)
    b = synth.normal_bf16((N, K), 2, std=0.02)
    ca, sa = oracle.quantize(a, oracle.LAYOUT_1D_ROW)
    cb, sb = oracle.quantize(b, oracle.LAYOUT_1D_ROW)
    c, s = oracle.gemm(ca, sa, cb, sb, K)
    A = _decode_tensor(ca, sa, K)
    B = _decode_tensor(cb, sb, K)
    ref = A @ B.T
    assert np.allclose(c, ref, rtol=1e-12, atol=1e-300)
    assert np.allclose(s, np.abs(A) @ np.abs(B).T, rtol=1e-12, atol=1e-300)
    assert np.all(s >= np.abs(c))
    cc, ss = oracle.gemm_entries(ca, sa, cb, sb, K, [(0, 0), (M - 1, N - 1), (M // 2, N // 3)])
    assert cc[0] == c[0, 0] and cc[1] == c[M - 1, N - 1] and ss[2] == s[M // 2, N // 3]


def test_gemm_nan_scale_propagates():
    a = synth.normal_bf16((4, 64), 1)
    b = synth.normal_bf16((3, 64), 2)
    ca, sa = oracle.quantize(a, oracle.LAYOUT_1D_ROW)
    cb, sb = oracle.quantize(b, oracle.LAYOUT_1D_ROW)
    sa[1, 1] = 0xFF
    c = oracle.gemm(ca, sa, cb, sb, 64, want_abs=False)
    assert np.all(np.isnan(c[1])) and not np.any(np.isnan(c[[0, 2, 3]]))


def test_gemm_2d_scale_modes():
    w = synth.normal_bf16((64, 96), 3, 0.02)
    x = synth.normal_bf16((8, 96), 4)
    cw, sw, cwt = oracle.quantize(w, oracle.LAYOUT_2D, transposed_copy=True)
    cx, sx = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    # fprop: X W^T with W's 2D scales
    c1 = oracle.gemm(cx, sx, cw, sw, 96, 0, 1, want_abs=False)
    ref = _decode_tensor(cx, sx, 96) @ _decode_tensor(cw, sw, 96, 1).T
    assert np.allclose(c1, ref, rtol=1e-12, atol=0)
    # dgrad-style: D W with W^T stored as the transposed copy, scales of W read transposed
    d = synth.normal_bf16((8, 64), 5)
    cd, sd = oracle.quantize(d, oracle.LAYOUT_1D_ROW)
    c2 = oracle.gemm(cd, sd, cwt, sw, 64, 0, 2, want_abs=False)
    Wdec = _decode_tensor(cw, sw, 96, 1)                  # [64, 96]
    ref2 = _decode_tensor(cd, sd, 64) @ Wdec
    assert np.allclose(c2, ref2, rtol=1e-12, atol=0)
