"""GPU parity: mxfp4_gemm / mxfp4_grouped_gemm through the C ABI against the fp64 oracle.

Tolerance (block dot products, "Conversion rules" on "MXFP4", FP32 result):
|C_gpu - C_fp64| <= 1e-5 * sum_k |a_k b_k| element-wise.  The tcgen05 MMA
accumulates each 64-element K step into FP32, so the FP32 rounding error is at
most (K/64) * 2^-24 * sum|a b| (<= 5.4e-6 * S for K = 5760) plus the
rounding inside a step, which the bound leaves room for.
"""
import numpy as np
import pytest
import torch

import oracle
import quantize_block_scaled_rht_b200 as mx
import synth
from mxfp4_testutil import assert_gemm_close, dev_bf16, dev_u8, expand_2d, from_mma, host, to_mma

pytestmark = pytest.mark.gpu


def _oracle_operand(bits, layout=oracle.LAYOUT_1D_ROW, rht=0, rnd=oracle.ROUND_RNE, seed=0):
    codes, scales = oracle.quantize(bits, layout, rht, rnd, seed)[:2]
    return codes, scales


def _run_gemm_from_oracle_operands(ca, sa, cb, sb, K):
    """GEMM on the GPU from oracle-quantized operands (scales moved to the MMA layout)."""
    out = mx.mxfp4_gemm(dev_u8(ca), dev_u8(to_mma(sa, K)), dev_u8(cb), dev_u8(to_mma(sb, K)), K)
    torch.cuda.synchronize()
    return host(out)


def test_pr1_256_cube_quantize_and_gemm_on_gpu():
    """PR1: X, Y 256x256 N(0,1) (seeds 0, 1), 1D RNE, C = X Y^T."""
    xb, yb = synth.pr1_inputs()
    qx = mx.mxfp4_quantize(dev_bf16(xb), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    qy = mx.mxfp4_quantize(dev_bf16(yb), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    c = host(mx.mxfp4_gemm(qx.codes, qx.scales, qy.codes, qy.scales, 256))
    ca, sa = _oracle_operand(xb)
    cb, sb = _oracle_operand(yb)
    assert np.array_equal(host(qx.codes), ca) and np.array_equal(host(qy.codes), cb)
    ref, s = oracle.gemm(ca, sa, cb, sb, 256)
    assert_gemm_close(c, ref, s)


@pytest.mark.parametrize("M,N,K", [(128, 192, 64), (300, 200, 320), (512, 768, 1024), (130, 72, 2880),
                                   (1, 8, 128), (257, 388, 576)])
def test_gemm_shapes(M, N, K):
    a = synth.normal_bf16((M, K), 10 + M)
    b = synth.normal_bf16((N, K), 20 + N, 0.02)
    ca, sa = _oracle_operand(a)
    cb, sb = _oracle_operand(b)
    c = _run_gemm_from_oracle_operands(ca, sa, cb, sb, K)
    ref, s = oracle.gemm(ca, sa, cb, sb, K)
    assert_gemm_close(c, ref, s)


def test_gemm_wide_dynamic_range_and_nan():
    M, N, K = 256, 384, 512
    g = np.random.default_rng(3)
    a = synth.bf16_bits((g.standard_normal((M, K)) * 2.0 ** g.integers(-30, 30, (M, 1))).astype(np.float32))
    b = synth.bf16_bits((g.standard_normal((N, K)) * 2.0 ** g.integers(-30, 30, (1, K))).astype(np.float32))
    ca, sa = _oracle_operand(a)
    cb, sb = _oracle_operand(b)
    sa = sa.copy(); sb = sb.copy()
    sa[5, 3] = 0xFF
    sb[7, 0] = 0xFF
    c = _run_gemm_from_oracle_operands(ca, sa, cb, sb, K)
    ref, s = oracle.gemm(ca, sa, cb, sb, K)
    assert np.all(np.isnan(c[5])) and np.all(np.isnan(c[:, 7]))
    assert_gemm_close(c, ref, s)


def test_fprop_dgrad_with_2d_weight_and_transposed_copy():
    """W quantized once in 2D; fprop uses W's codes, dgrad the transposed copy."""
    T, H, I = 256, 320, 448
    x = synth.activations_with_outliers(T, H, seed=2)
    w = synth.normal_bf16((I, H), 3, 0.02)
    dy = synth.normal_bf16((T, I), 4, 1e-3)
    qw = mx.mxfp4_quantize(dev_bf16(w), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA, transposed_copy=True)
    qx = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    qdy = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_ROW, 0, mx.ROUND_SR, 42, scale_layout=mx.SCALES_MMA)
    y = host(mx.mxfp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, H))
    dx = host(mx.mxfp4_gemm(qdy.codes, qdy.scales, qw.codes_t, qw.scales_t, I))
    cw, sw, cwt = oracle.quantize(w, oracle.LAYOUT_2D, transposed_copy=True)
    cx, sx = _oracle_operand(x)
    cdy, sdy = _oracle_operand(dy, rnd=oracle.ROUND_SR, seed=42)
    ref_y, s_y = oracle.gemm(cx, sx, cw, sw, H, 0, 1)
    ref_dx, s_dx = oracle.gemm(cdy, sdy, cwt, sw, I, 0, 2)
    assert_gemm_close(y, ref_y, s_y)
    assert_gemm_close(dx, ref_dx, s_dx)


def test_wgrad_rht32_along_tokens():
    """wgrad: dY^T and X^T quantized along tokens (1D col) with RHT32 and shared signs."""
    T, H, I = 512, 192, 320
    x = synth.normal_bf16((T, H), 5)
    dy = synth.normal_bf16((T, I), 6, 1e-3)
    qdyt = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_COL, 32, mx.ROUND_SR, 42, scale_layout=mx.SCALES_MMA)
    qxt = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_COL, 32, mx.ROUND_RNE, 42, scale_layout=mx.SCALES_MMA)
    dw = host(mx.mxfp4_gemm(qdyt.codes, qdyt.scales, qxt.codes, qxt.scales, T))
    ca, sa = oracle.quantize(dy, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_SR, 42)
    cb, sb = oracle.quantize(x, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_RNE, 42)
    ref, s = oracle.gemm(ca, sa, cb, sb, T)
    assert_gemm_close(dw, ref, s)


def _grouped_case(sizes, N, K, seed=0):
    G = len(sizes)
    sizes = np.asarray(sizes, np.int32)
    padded = (sizes + 127) // 128 * 128
    offsets = np.zeros(G + 1, np.int32)
    offsets[1:] = np.cumsum(padded)
    rows = int(max(offsets[-1], 128))
    a = synth.normal_bf16((rows, K), seed + 1)
    w = synth.normal_bf16((G, N, K), seed + 2, 0.02)
    return sizes, offsets, rows, a, w


@pytest.mark.parametrize("sizes,N,K", [([1, 130, 0, 257, 128], 192, 256), ([300, 5, 64], 384, 576),
                                       ([17], 224, 128)])
def test_grouped_gemm(sizes, N, K):
    sizes, offsets, rows, a, w = _grouped_case(sizes, N, K)
    G = len(sizes)
    qa = mx.mxfp4_quantize(dev_bf16(a), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    qw = [mx.mxfp4_quantize(dev_bf16(w[g]), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA) for g in range(G)]
    b_codes = torch.stack([q.codes for q in qw])
    b_scales = torch.cat([q.scales for q in qw])
    sentinel = 12345.0
    out = torch.full((rows, N), sentinel, dtype=torch.float32, device="cuda")
    mx.mxfp4_grouped_gemm(qa.codes, qa.scales, torch.from_numpy(offsets).cuda(), torch.from_numpy(sizes).cuda(),
                          b_codes, b_scales, N, K, out=out)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    c = host(out)
    ca, sa = oracle.quantize(a, oracle.LAYOUT_1D_ROW)
    for g in range(G):
        o, n = int(offsets[g]), int(sizes[g])
        cw, sw = oracle.quantize(w[g], oracle.LAYOUT_2D)
        if n:
            ref, s = oracle.gemm(ca[o:o + n], sa[o:o + n], cw, sw, K, 0, 1)
            assert_gemm_close(c[o:o + n], ref, s)
        # padding rows of the group are never written
        assert np.all(c[o + n:int(offsets[g + 1])] == sentinel)


def test_grouped_gemm_misaligned_offset_is_reported():
    sizes, offsets, rows, a, w = _grouped_case([64, 64], 192, 128)
    offsets = offsets.copy()
    offsets[1] = 100                                        # not a multiple of 128
    qa = mx.mxfp4_quantize(dev_bf16(a), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    qw = [mx.mxfp4_quantize(dev_bf16(w[g]), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA) for g in range(2)]
    mx.mxfp4_grouped_gemm(qa.codes, qa.scales, torch.from_numpy(offsets).cuda(), torch.from_numpy(sizes).cuda(),
                          torch.stack([q.codes for q in qw]), torch.cat([q.scales for q in qw]), 192, 128)
    assert mx.mxfp4_get_error() == mx.MXFP4_ERR_INVALID_ARG
    assert mx.mxfp4_get_error() == mx.MXFP4_OK


def test_gemm_rejects_bad_k_and_alignment():
    a = torch.zeros((128, 48), dtype=torch.uint8, device="cuda")
    s = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(mx.MXFP4Error) as e:
        mx.mxfp4_gemm(a, s, a, s, 96)                       # K % 64 != 0
    assert e.value.status == mx.MXFP4_ERR_UNSUPPORTED
    big = torch.zeros((128, 80), dtype=torch.uint8, device="cuda")
    with pytest.raises(mx.MXFP4Error) as e:
        mx.mxfp4_gemm(big[:, 8:], s, big[:, 8:], s, 128)    # misaligned pointer
    assert e.value.status == mx.MXFP4_ERR_ALIGNMENT


def test_bounded_wait_reports_timeout_and_context_survives():
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    mx.mxfp4_wait_probe(True)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    old = mx.mxfp4_set_wait_limit_ns(2_000_000)             # 2 ms
    try:
        mx.mxfp4_wait_probe(False)                          # nothing ever arrives
        assert mx.mxfp4_get_error() == mx.MXFP4_ERR_TIMEOUT
    finally:
        mx.mxfp4_set_wait_limit_ns(old)
    # the context is still usable
    test_gemm_shapes(128, 192, 64)


def _routed_wgrad_case(sizes, M, N, seed):
    """Expert-sorted routed tensors dY [K, M] and X [K, N] with groups padded
    to 128 rows (padding rows zero), and the offsets along K."""
    g = np.random.default_rng(seed)
    padded = [((s + 127) // 128) * 128 for s in sizes]
    offsets = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    K = int(offsets[-1])
    dy = np.zeros((K, M), np.float32)
    x = np.zeros((K, N), np.float32)
    for e, s in enumerate(sizes):
        o = offsets[e]
        dy[o:o + s] = g.standard_normal((s, M)) * 1e-3
        x[o:o + s] = g.standard_normal((s, N))
    return synth.bf16_bits(dy), synth.bf16_bits(x), offsets, K


@pytest.mark.parametrize("sizes", [[200, 0, 513, 128], [1024], [0, 0, 300]])
def test_grouped_wgrad_matches_oracle(sizes):
    M, N = 320, 224
    dy, x, offsets, K = _routed_wgrad_case(sizes, M, N, seed=len(sizes) + sum(sizes))
    qa = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_COL, 32, mx.ROUND_SR, 42, scale_layout=mx.SCALES_MMA)
    qb = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_COL, 32, mx.ROUND_RNE, 42, scale_layout=mx.SCALES_MMA)
    c = mx.mxfp4_grouped_gemm_wgrad(qa.codes, qa.scales, qb.codes, qb.scales,
                                    torch.from_numpy(offsets).cuda(), K)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    c = host(c)
    ca, sa = oracle.quantize(dy, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_SR, 42)
    cb, sb = oracle.quantize(x, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_RNE, 42)
    for e in range(len(sizes)):
        o0, o1 = int(offsets[e]), int(offsets[e + 1])
        ce = c[e * M:(e + 1) * M]
        if o1 == o0:
            assert np.all(ce == 0.0)
            continue
        ref, s = oracle.gemm(ca[:, o0 // 2:o1 // 2], sa[:, o0 // 32:o1 // 32], cb[:, o0 // 2:o1 // 2],
                             sb[:, o0 // 32:o1 // 32], o1 - o0)
        assert_gemm_close(ce.astype(np.float64), ref, s)


def test_grouped_wgrad_bad_offset_reported():
    M, N = 128, 128
    dy, x, offsets, K = _routed_wgrad_case([128, 128], M, N, seed=3)
    qa = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_COL, scale_layout=mx.SCALES_MMA)
    qb = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_COL, scale_layout=mx.SCALES_MMA)
    bad = torch.tensor([0, 64, 256], dtype=torch.int32, device="cuda")
    mx.mxfp4_grouped_gemm_wgrad(qa.codes, qa.scales, qb.codes, qb.scales, bad, K)
    assert mx.mxfp4_get_error() == mx.MXFP4_ERR_INVALID_ARG


def test_grouped_dgrad_with_transposed_weight_copies():
    """MoE dgrad: dX_e = dY_e W_e, with B_e the 2D transposed copy of expert
    e's weight (W and W^T share one quantization)."""
    sizes, I, H = [100, 0, 260], 256, 192
    g = np.random.default_rng(11)
    padded = [((s + 127) // 128) * 128 for s in sizes]
    offsets = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    rows = int(offsets[-1])
    dy = np.zeros((rows, I), np.float32)
    for e, s in enumerate(sizes):
        dy[offsets[e]:offsets[e] + s] = g.standard_normal((s, I)) * 1e-3
    dy = synth.bf16_bits(dy)
    ws = [synth.normal_bf16((I, H), 30 + e, 0.02) for e in range(len(sizes))]
    qa = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_ROW, 0, mx.ROUND_SR, 42, scale_layout=mx.SCALES_MMA)
    qw = [mx.mxfp4_quantize(dev_bf16(w), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA, transposed_copy=True) for w in ws]
    c = mx.mxfp4_grouped_gemm(qa.codes, qa.scales, torch.from_numpy(offsets).cuda(),
                              torch.tensor(sizes, dtype=torch.int32, device="cuda"),
                              torch.stack([q.codes_t for q in qw]), torch.cat([q.scales_t for q in qw]), H, I)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    c = host(c)
    ca, sa = oracle.quantize(dy, oracle.LAYOUT_1D_ROW, 0, oracle.ROUND_SR, 42)
    for e, s in enumerate(sizes):
        if s == 0:
            continue
        cw, sw, cwt = oracle.quantize(ws[e], oracle.LAYOUT_2D, transposed_copy=True)
        o = int(offsets[e])
        pairs = [(o + r, n) for r in range(0, s, 7) for n in range(0, H, 5)] + [(o + s - 1, H - 1)]
        ref, sabs = oracle.gemm_entries(ca, sa, cwt, sw, I, pairs, 0, 2)
        got = np.array([c[m, n] for m, n in pairs], np.float64)
        assert_gemm_close(got, ref, sabs)


@pytest.mark.parametrize("shape", [(256, 192, 256), (304, 208, 576), (512, 384, 1024)])
def test_nvfp4_gemm_matches_oracle(shape):
    M, N, K = shape
    a = synth.normal_bf16((M, K), 40)
    b = synth.normal_bf16((N, K), 41, 0.02)
    qa = mx.mxfp4_nvfp4_quantize(dev_bf16(a), scale_layout=mx.SCALES_MMA)
    qb = mx.mxfp4_nvfp4_quantize(dev_bf16(b), scale_layout=mx.SCALES_MMA)
    c = host(mx.mxfp4_nvfp4_gemm(qa, qb))
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    ca, sa, aa = oracle.nvfp4_quantize(a, oracle.LAYOUT_1D_ROW)
    cb, sb, ab = oracle.nvfp4_quantize(b, oracle.LAYOUT_1D_ROW)
    g = np.random.default_rng(M + N)
    pairs = list(zip(g.integers(0, M, 400), g.integers(0, N, 400))) + [(0, 0), (M - 1, N - 1)]
    ref, s = oracle.nvfp4_gemm_entries(ca, sa, aa, cb, sb, ab, K, pairs)
    got = np.array([c[m, n] for m, n in pairs], np.float64)
    assert_gemm_close(got, ref, s)


def _assert_bf16_close(c16: np.ndarray, ref: np.ndarray, s: np.ndarray):
    """bf16 output: the FP32 bound of assert_gemm_close plus one bf16 rounding
    of the FP32 value (8 significant bits, so round to nearest is within
    2^-8 of the value)."""
    nan_ref = np.isnan(ref)
    assert np.array_equal(np.isnan(c16), nan_ref)
    ok = ~nan_ref
    err = np.abs(c16[ok].astype(np.float64) - ref[ok])
    fp32_bound = 1e-5 * s[ok]
    bound = fp32_bound + 2.0 ** -8 * (np.abs(ref[ok]) + fp32_bound)
    assert not (err > bound).any(), f"{int((err > bound).sum())} entries outside the bf16 bound"


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("M,N,K", [(128, 192, 64), (300, 200, 320), (1, 8, 128), (257, 392, 576),
                                   (512, 768, 1024), (130, 72, 2880)])
def test_gemm_bf16_output(M, N, K):
    """bf16 epilogue: within the oracle bound, and bit-equal to the RNE of the
    FP32 path's output for the same operands (same accumulators)."""
    a = synth.normal_bf16((M, K), 30 + M)
    b = synth.normal_bf16((N, K), 40 + N, 0.02)
    ca, sa = _oracle_operand(a)
    cb, sb = _oracle_operand(b)
    args = (dev_u8(ca), dev_u8(to_mma(sa, K)), dev_u8(cb), dev_u8(to_mma(sb, K)), K)
    c16 = mx.mxfp4_gemm_bf16(*args)
    c32 = mx.mxfp4_gemm(*args)
    torch.cuda.synchronize()
    assert np.array_equal(_bf16_bits(c16), _bf16_bits(c32.to(torch.bfloat16)))
    ref, s = oracle.gemm(ca, sa, cb, sb, K)
    _assert_bf16_close(c16.float().cpu().numpy(), ref, s)


def test_gemm_bf16_nan_and_strided_output():
    """NaN scales give NaN rows/columns; a wider output row stride leaves the
    columns past N untouched."""
    M, N, K = 256, 200, 256
    a = synth.normal_bf16((M, K), 7)
    b = synth.normal_bf16((N, K), 8, 0.02)
    ca, sa = _oracle_operand(a)
    cb, sb = _oracle_operand(b)
    sa = sa.copy(); sa[3, 1] = 0xFF
    big = torch.full((M, N + 24), 77.0, dtype=torch.bfloat16, device="cuda")
    out = big[:, :N]
    mx.mxfp4_gemm_bf16(dev_u8(ca), dev_u8(to_mma(sa, K)), dev_u8(cb), dev_u8(to_mma(sb, K)), K, out=out)
    torch.cuda.synchronize()
    c = out.float().cpu().numpy()
    assert np.all(np.isnan(c[3]))
    assert torch.all(big[:, N:] == 77.0)
    ref, s = oracle.gemm(ca, sa, cb, sb, K)
    _assert_bf16_close(c, ref, s)


@pytest.mark.parametrize("sizes,N,K", [([1, 130, 0, 257, 128], 192, 256), ([300, 5, 64], 384, 576),
                                       ([17], 224, 128)])
def test_grouped_gemm_bf16(sizes, N, K):
    sizes, offsets, rows, a, w = _grouped_case(sizes, N, K)
    G = len(sizes)
    qa = mx.mxfp4_quantize(dev_bf16(a), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    qw = [mx.mxfp4_quantize(dev_bf16(w[g]), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA) for g in range(G)]
    b_codes = torch.stack([q.codes for q in qw])
    b_scales = torch.cat([q.scales for q in qw])
    d_off, d_sz = torch.from_numpy(offsets).cuda(), torch.from_numpy(sizes).cuda()
    out16 = torch.full((rows, N), 1280.0, dtype=torch.bfloat16, device="cuda")
    mx.mxfp4_grouped_gemm_bf16(qa.codes, qa.scales, d_off, d_sz, b_codes, b_scales, N, K, out=out16)
    out32 = torch.full((rows, N), 1280.0, dtype=torch.float32, device="cuda")
    mx.mxfp4_grouped_gemm(qa.codes, qa.scales, d_off, d_sz, b_codes, b_scales, N, K, out=out32)
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    # the padding rows keep 1280 (exact in bf16) in both; every written entry is the RNE of the FP32 one
    assert np.array_equal(_bf16_bits(out16), _bf16_bits(out32.to(torch.bfloat16)))
    c = out16.float().cpu().numpy()
    ca, sa = oracle.quantize(a, oracle.LAYOUT_1D_ROW)
    for g in range(G):
        o, n = int(offsets[g]), int(sizes[g])
        if n:
            cw, sw = oracle.quantize(w[g], oracle.LAYOUT_2D)
            ref, s = oracle.gemm(ca[o:o + n], sa[o:o + n], cw, sw, K, 0, 1)
            _assert_bf16_close(c[o:o + n], ref, s)
        assert np.all(c[o + n:int(offsets[g + 1])] == 1280.0)


# --- MXFP4-output epilogue ------------------------------------------------------
_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _scale_code(amax: np.ndarray) -> np.ndarray:
    """E8M0 code of the reference rule for finite amax >= 0 (0 -> 0):
    floor(log2 amax) - 2 + 127, the exponent taken exactly by frexp."""
    _, e = np.frexp(np.where(amax > 0, amax, 1.0))
    return np.where(amax > 0, np.clip(e.astype(np.int64) - 1 - 2 + 127, 0, 254), 0).astype(np.int64)


def _rne_value(y: np.ndarray) -> np.ndarray:
    """Signed E2M1 value nearest to y (ties to the even code), saturating at 6."""
    a = np.minimum(np.abs(y), 6.0)
    d = np.abs(a[..., None] - _GRID) + (np.arange(8) % 2) * 1e-9
    return np.sign(y) * _GRID[np.argmin(d, axis=-1)]


def _decode(codes: np.ndarray) -> np.ndarray:
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    return np.where(nib & 8, -1.0, 1.0) * _GRID[nib & 7]


def _requantize_f32(c32: np.ndarray):
    """Test-side 1D-row requantization of FP32 values (reference scale rule,
    RNE): the scaled values are formed in fp32 as the kernels form them."""
    M, N = c32.shape
    blk = c32.reshape(M, N // 32, 32)
    amax = np.abs(blk).max(axis=-1).astype(np.float64)
    sc = _scale_code(amax)
    inv = np.ldexp(np.float32(1.0), (127 - sc).astype(np.int32)).astype(np.float32)
    y = (blk * inv[..., None]).astype(np.float32)
    return _rne_value(y.astype(np.float64)).reshape(M, N), sc


@pytest.mark.parametrize("M,N,K", [(256, 192, 512), (300, 224, 320), (130, 384, 2880)])
@pytest.mark.parametrize("mma", [False, True])
def test_gemm_mxfp4_output(M, N, K, mma):
    """MXFP4-output epilogue: (1) bit-equal to the 1D-row RNE requantization
    of the FP32 kernel's own product; (2) every scale and element code is one
    that an FP32 product within 1e-5 * sum|ab| of the exact one can give."""
    a = synth.normal_bf16((M, K), 50 + M)
    b = synth.normal_bf16((N, K), 60 + N, 0.02)
    ca, sa = _oracle_operand(a)
    cb, sb = _oracle_operand(b)
    args = (dev_u8(ca), dev_u8(to_mma(sa, K)), dev_u8(cb), dev_u8(to_mma(sb, K)), K)
    sl = mx.SCALES_MMA if mma else mx.SCALES_ROWMAJOR
    q = mx.mxfp4_gemm_mxfp4(*args, scale_layout=sl)
    c32 = mx.mxfp4_gemm(*args)
    torch.cuda.synchronize()
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    sc = host(q.scales)
    sc = from_mma(sc, M, N) if mma else sc
    got = _decode(host(q.codes)) * np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32, axis=1)
    # (1) the same accumulators, requantized on the host
    want_v, want_sc = _requantize_f32(host(c32))
    assert np.array_equal(sc, want_sc)
    assert np.array_equal(_decode(host(q.codes)), want_v)
    # (2) against the exact product, within the GEMM tolerance
    ref, s = oracle.gemm(ca, sa, cb, sb, K)
    tol = 1e-5 * s
    blk = lambda x: x.reshape(M, N // 32, 32)
    amax_lo = np.maximum(np.abs(blk(ref)) - blk(tol), 0).max(axis=-1)
    amax_hi = (np.abs(blk(ref)) + blk(tol)).max(axis=-1)
    assert np.all((_scale_code(amax_lo) <= sc) & (sc <= _scale_code(amax_hi)))
    X = np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32, axis=1)
    lo, hi = _rne_value((ref - tol) / X) * X, _rne_value((ref + tol) / X) * X
    assert np.all((lo <= got) & (got <= hi))
    assert np.mean(lo == hi) > 0.99          # almost every code is fixed by the exact product


def test_gemm_mxfp4_output_nan_rows():
    M, N, K = 128, 192, 256
    a = synth.normal_bf16((M, K), 3)
    b = synth.normal_bf16((N, K), 4, 0.02)
    ca, sa = _oracle_operand(a)
    cb, sb = _oracle_operand(b)
    sa = sa.copy(); sa[9, 2] = 0xFF
    q = mx.mxfp4_gemm_mxfp4(dev_u8(ca), dev_u8(to_mma(sa, K)), dev_u8(cb), dev_u8(to_mma(sb, K)), K)
    torch.cuda.synchronize()
    sc, codes = host(q.scales), host(q.codes)
    assert np.all(sc[9] == 0xFF) and np.all(codes[9] == 0)
    assert np.all(np.delete(sc, 9, axis=0) != 0xFF)


@pytest.mark.parametrize("sizes", [[200, 0, 513, 128], [0, 0, 300]])
def test_grouped_wgrad_bf16(sizes):
    """bf16 grouped wgrad: bit-equal to the RNE of the FP32 grouped wgrad on
    the same operands (empty groups zero)."""
    M, N = 320, 224
    dy, x, offsets, K = _routed_wgrad_case(sizes, M, N, seed=len(sizes) + sum(sizes))
    qa = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_COL, 32, mx.ROUND_SR, 42, scale_layout=mx.SCALES_MMA)
    qb = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_COL, 32, mx.ROUND_RNE, 42, scale_layout=mx.SCALES_MMA)
    off = torch.from_numpy(offsets).cuda()
    c32 = mx.mxfp4_grouped_gemm_wgrad(qa.codes, qa.scales, qb.codes, qb.scales, off, K)
    c16 = mx.mxfp4_grouped_gemm_wgrad_bf16(qa.codes, qa.scales, qb.codes, qb.scales, off, K)
    torch.cuda.synchronize()
    assert mx.mxfp4_get_error() == mx.MXFP4_OK
    assert torch.equal(c16.view(torch.int16), c32.to(torch.bfloat16).view(torch.int16))


@pytest.mark.parametrize("rows,k,two_d", [(256, 2880, False), (130, 320, False), (1, 64, False),
                                          (192, 2880, True), (96, 576, True)])
def test_scales_to_mma_matches_host_permutation(rows, k, two_d):
    """mxfp4_scales_to_mma writes every valid (row, K-block) byte where the
    GEMM-ready layout puts it (2D tile scales repeated on their 32 rows) and
    zero in every pad byte."""
    g = np.random.default_rng(rows + k)
    srows = rows // 32 if two_d else rows
    canon = g.integers(0, 256, size=(srows, k // 32), dtype=np.uint8)
    out = dev_u8(np.full(mx.mma_scales_bytes(rows, k), 0xA5, np.uint8))
    mx.mxfp4_scales_to_mma(dev_u8(canon), rows, k, two_d=two_d, out=out)
    got = host(out)
    per_row = expand_2d(canon, rows) if two_d else canon
    assert np.array_equal(got, to_mma(per_row, k))   # to_mma zero-fills the pads


def test_gemm_from_canonical_2d_weight_scales():
    """A caller holding canonical scales (1D row-major for X, 2D tile scales for
    W) converts them with mxfp4_scales_to_mma and gets the same products as
    from the quantizer's GEMM-ready scales, bit for bit."""
    T, H, I = 256, 576, 384
    x = synth.activations_with_outliers(T, H, seed=2)
    w = synth.normal_bf16((I, H), 3, 0.02)
    qx_rm = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_ROW)
    qw_rm = mx.mxfp4_quantize(dev_bf16(w), mx.LAYOUT_2D, transposed_copy=True)
    qx = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    qw = mx.mxfp4_quantize(dev_bf16(w), mx.LAYOUT_2D, scale_layout=mx.SCALES_MMA, transposed_copy=True)
    sx = mx.mxfp4_scales_to_mma(qx_rm.scales, T, H)
    sw = mx.mxfp4_scales_to_mma(qw_rm.scales, I, H, two_d=True)
    swt = mx.mxfp4_scales_to_mma(qw_rm.scales_t, H, I, two_d=True)
    c_ref = host(mx.mxfp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, H))
    c = host(mx.mxfp4_gemm(qx_rm.codes, sx, qw_rm.codes, sw, H))
    assert np.array_equal(c.view(np.uint32), c_ref.view(np.uint32))
    # dgrad-style product through the transposed copy and its converted tile scales
    dy = synth.normal_bf16((T, I), 4, 1e-3)
    qdy = mx.mxfp4_quantize(dev_bf16(dy), mx.LAYOUT_1D_ROW, scale_layout=mx.SCALES_MMA)
    d_ref = host(mx.mxfp4_gemm(qdy.codes, qdy.scales, qw.codes_t, qw.scales_t, I))
    d = host(mx.mxfp4_gemm(qdy.codes, qdy.scales, qw_rm.codes_t, swt, I))
    assert np.array_equal(d.view(np.uint32), d_ref.view(np.uint32))
