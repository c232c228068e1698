"""GPU parity: mxfp4_quantize / mxfp4_dequantize through the C ABI against the oracle.

Codes and scales must be bit-exact (including stochastic rounding and the RHT).
Shapes span several CTA tiles with ragged tails; edge cases cover every bf16
bit pattern (NaN, Inf, subnormals, zeros, ties, saturation).
"""
import numpy as np
import pytest
import torch

import oracle
import quantize_block_scaled_rht_b200 as mx
import synth
from mxfp4_testutil import dev_bf16, expand_2d, from_mma, host

pytestmark = pytest.mark.gpu

LAYOUTS = [mx.LAYOUT_1D_ROW, mx.LAYOUT_1D_COL, mx.LAYOUT_2D]
SHAPES = {mx.LAYOUT_1D_ROW: (67, 352), mx.LAYOUT_1D_COL: (288, 136), mx.LAYOUT_2D: (96, 288)}


def _quantize_both(x_bits, layout, rht, rnd, seed, scale_layout, offset=0, trans=False):
    x = dev_bf16(x_bits)
    q = mx.mxfp4_quantize(x, layout, rht, rnd, seed, offset, scale_layout, transposed_copy=trans)
    torch.cuda.synchronize()
    ref = oracle.quantize(x_bits, layout, rht, rnd, seed, offset, transposed_copy=trans)
    return q, ref


def _scales_rowmajor(q, layout, ref_scales, rows, cols):
    s = host(q.scales)
    if q.scale_layout == mx.SCALES_ROWMAJOR:
        return s
    if layout == mx.LAYOUT_2D:
        return from_mma(s, rows, cols)      # per-row expansion of the tile scales
    return from_mma(s, q.rows, q.k)


@pytest.mark.parametrize("scale_layout", [mx.SCALES_ROWMAJOR, mx.SCALES_MMA])
@pytest.mark.parametrize("rnd", [mx.ROUND_RNE, mx.ROUND_SR])
@pytest.mark.parametrize("rht", [0, 16, 32])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_quantize_bit_exact(layout, rht, rnd, scale_layout):
    rows, cols = SHAPES[layout]
    x = synth.student_t_bf16((rows, cols), seed=100 + layout * 7 + rht)
    trans = layout == mx.LAYOUT_2D
    q, ref = _quantize_both(x, layout, rht, rnd, 42, scale_layout, trans=trans)
    assert np.array_equal(host(q.codes), ref[0])
    got = _scales_rowmajor(q, layout, ref[1], rows, cols)
    want = expand_2d(ref[1], rows) if (layout == mx.LAYOUT_2D and scale_layout == mx.SCALES_MMA) else ref[1]
    assert np.array_equal(got, want)
    if trans:
        assert np.array_equal(host(q.codes_t), ref[2])
        st = host(q.scales_t)
        if scale_layout == mx.SCALES_ROWMAJOR:
            assert np.array_equal(st, ref[1].T)
        else:
            assert np.array_equal(from_mma(st, cols, rows), expand_2d(ref[1].T, cols))


@pytest.mark.parametrize("scale_layout", [mx.SCALES_ROWMAJOR, mx.SCALES_MMA])
@pytest.mark.parametrize("rht,rnd", [(0, mx.ROUND_RNE), (32, mx.ROUND_RNE), (32, mx.ROUND_SR)])
def test_column_quantizer_strips(rht, rnd, scale_layout):
    """1D-column quantization of 65,632 x 1080: 257 row tiles of 256 (the last
    holds 96 rows, so 3 of its 8 K-blocks), 17 column tiles of 64 (the last
    holds 56 columns).  With 148 SMs the launcher walks strips of 4 vertically
    adjacent tiles whose scales leave together, so the last strip is one
    ragged tile; the scale rows (2051 bytes) are not word-aligned, so the
    row-major scales leave byte by byte.  Codes and scales must be bit-exact,
    under SR too (each element's stream index is its position in the
    transposed view)."""
    rows, cols = 65632, 1080
    x = synth.student_t_bf16((rows, cols), seed=12)
    q = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_COL, rht, rnd, 42, 0, scale_layout)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_COL, rht, rnd, 42)[:2]
    assert np.array_equal(host(q.codes), codes)
    assert np.array_equal(_scales_rowmajor(q, mx.LAYOUT_1D_COL, scales, rows, cols), scales)


@pytest.mark.parametrize("rht", [0, 32])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_every_bf16_pattern(layout, rht):
    """All 65536 bf16 bit patterns, in blocks, twice: as they come (each block
    scaled by its own max) and with a 4.0 in every row block (scale 1)."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    g = np.random.default_rng(5)
    a = g.permutation(allbits).reshape(256, 256)
    b = a.copy()
    b[:, ::32] = 0x4080                                   # 4.0
    x = np.concatenate([a, b], axis=0)
    for rnd in (mx.ROUND_RNE, mx.ROUND_SR):
        q, ref = _quantize_both(x, layout, rht, rnd, 9, mx.SCALES_ROWMAJOR, trans=(layout == mx.LAYOUT_2D))
        assert np.array_equal(host(q.codes), ref[0])
        assert np.array_equal(host(q.scales), ref[1])
        if layout == mx.LAYOUT_2D:
            assert np.array_equal(host(q.codes_t), ref[2])


def test_adversarial_blocks():
    vals = np.zeros((8, 64), np.float32)
    vals[0, :32] = 7.5; vals[0, 1] = 0.25; vals[0, 2] = -0.75; vals[0, 3] = 5.0
    vals[1, :32] = np.linspace(-6, 6, 32)
    vals[1, 32:] = [0.25 * i for i in range(32)]           # ties after scaling
    vals[2, :] = 3.3895314e38                               # near bf16 max
    vals[3, :32] = np.float32(2.0 ** -133)                  # bf16 subnormals
    vals[3, 32:] = -0.0
    vals[4, :] = [8.0, -8.0] * 32
    vals[5, :32] = 6.0; vals[5, 32:] = 1e-30
    x = synth.bf16_bits(vals)
    x[6, 5] = 0x7FC0                                        # NaN
    x[7, 40] = 0xFF80                                       # -Inf
    for layout in (mx.LAYOUT_1D_ROW,):
        for rht in (0, 16, 32):
            for rnd in (mx.ROUND_RNE, mx.ROUND_SR):
                q, ref = _quantize_both(x, layout, rht, rnd, 3, mx.SCALES_ROWMAJOR)
                assert np.array_equal(host(q.codes), ref[0]), (rht, rnd)
                assert np.array_equal(host(q.scales), ref[1]), (rht, rnd)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_sharded_sr_equals_whole(layout):
    rows, cols = 256, 192
    x = synth.student_t_bf16((rows, cols), seed=77)
    whole = mx.mxfp4_quantize(dev_bf16(x), layout, 32, mx.ROUND_SR, 42)
    if layout == mx.LAYOUT_1D_COL:
        pa = mx.mxfp4_quantize(dev_bf16(np.ascontiguousarray(x[:, :96])), layout, 32, mx.ROUND_SR, 42, 0)
        pb = mx.mxfp4_quantize(dev_bf16(np.ascontiguousarray(x[:, 96:])), layout, 32, mx.ROUND_SR, 42, 96 * rows)
    else:
        pa = mx.mxfp4_quantize(dev_bf16(np.ascontiguousarray(x[:128])), layout, 32, mx.ROUND_SR, 42, 0)
        pb = mx.mxfp4_quantize(dev_bf16(np.ascontiguousarray(x[128:])), layout, 32, mx.ROUND_SR, 42, 128 * cols)
    assert torch.equal(whole.codes, torch.cat([pa.codes, pb.codes]))
    assert torch.equal(whole.scales, torch.cat([pa.scales, pb.scales]))


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rht", [0, 16, 32])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_dequantize_matches_oracle(layout, rht, out_dtype):
    rows, cols = SHAPES[layout]
    x = synth.student_t_bf16((rows, cols), seed=300 + layout)
    codes, scales = oracle.quantize(x, layout, rht, oracle.ROUND_SR, 11)[:2]
    scales = scales.copy()
    scales.reshape(-1)[3] = 0xFF                            # one NaN block
    f32, b16 = oracle.dequantize(codes, scales, rows, cols, layout, rht, 11)
    out = mx.mxfp4_dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), rows, cols,
                              layout, rht, 11, out_dtype=out_dtype)
    got = host(out)
    if out_dtype == torch.float32:
        assert np.array_equal(np.isnan(got), np.isnan(f32))
        ok = ~np.isnan(f32)
        assert np.array_equal(got[ok].view(np.uint32), f32[ok].view(np.uint32))
    else:
        nan = np.isnan(synth.bf16_to_f32(b16))
        assert np.array_equal(np.isnan(synth.bf16_to_f32(got)), nan)
        assert np.array_equal(got[~nan], b16[~nan])


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rht", [16, 32])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_dequantize_rht_every_scale_code(layout, rht, out_dtype):
    """The inverse RHT over random codes with every scale code 0..255: the
    dequantizers transform scale codes 27..246 in the unscaled domain and the
    others (subnormal, overflowing and NaN scales) directly; both must equal
    the oracle's scaled butterfly bit for bit (NaN positions equal)."""
    rows, cols = {mx.LAYOUT_1D_ROW: (256, 320), mx.LAYOUT_1D_COL: (320, 256), mx.LAYOUT_2D: (512, 512)}[layout]
    rng = np.random.default_rng(900 + layout * 10 + rht)
    if layout == mx.LAYOUT_1D_COL:
        codes = rng.integers(0, 256, size=(cols, rows // 2), dtype=np.uint8)
        sshape = (cols, rows // 32)
    else:
        codes = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
        sshape = (rows // 32, cols // 32) if layout == mx.LAYOUT_2D else (rows, cols // 32)
    n = sshape[0] * sshape[1]
    scales = rng.permutation(np.arange(n) % 256).astype(np.uint8).reshape(sshape)
    assert len(np.unique(scales)) == 256
    f32, b16 = oracle.dequantize(codes, scales, rows, cols, layout, rht, 5)
    out = mx.mxfp4_dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), rows, cols,
                              layout, rht, 5, out_dtype=out_dtype)
    got = host(out)
    if out_dtype == torch.float32:
        assert np.array_equal(np.isnan(got), np.isnan(f32))
        ok = ~np.isnan(f32)
        assert np.array_equal(got[ok].view(np.uint32), f32[ok].view(np.uint32))
    else:
        nan = np.isnan(synth.bf16_to_f32(b16))
        assert np.array_equal(np.isnan(synth.bf16_to_f32(got)), nan)
        assert np.array_equal(got[~nan], b16[~nan])


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rht", [16, 32])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_dequantize_rht_signed_zeros(layout, rht, out_dtype):
    """Blocks built to make the inverse butterfly produce exact zeros: all
    codes +-0 (codes 0 and 8), a +-0 first half with +-0.5 after it, and +-0
    / +-0.5 throughout.  The sign of an exact zero depends on the butterfly's
    order and pairing, which the dequantizers must follow exactly; every
    output bit pattern, zero signs included, must equal the oracle's."""
    rows, cols = {mx.LAYOUT_1D_ROW: (256, 320), mx.LAYOUT_1D_COL: (320, 256), mx.LAYOUT_2D: (512, 512)}[layout]
    rng = np.random.default_rng(1700 + layout * 10 + rht)
    if layout == mx.LAYOUT_1D_COL:
        shape, sshape = (cols, rows // 2), (cols, rows // 32)
    else:
        shape = (rows, cols // 2)
        sshape = (rows // 32, cols // 32) if layout == mx.LAYOUT_2D else (rows, cols // 32)
    nblk = shape[0] * shape[1] // 16
    nib = rng.choice(np.array([0, 8], dtype=np.uint8), size=(nblk, 32))     # every element +-0
    kind = rng.integers(0, 3, size=nblk)
    small = rng.choice(np.array([0, 1, 8, 9], dtype=np.uint8), size=(nblk, 32))   # +-0, +-0.5
    nib[kind == 1, 16:] = small[kind == 1, 16:]
    nib[kind == 2] = small[kind == 2]
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8).reshape(shape)
    # scale codes mostly in the unscaled-domain range, some outside it (no NaN)
    scales = rng.integers(100, 150, size=sshape).astype(np.uint8)
    edge = rng.random(sshape) < 0.1
    scales[edge] = rng.choice(np.array([0, 1, 20, 26, 247, 254], dtype=np.uint8), size=int(edge.sum()))
    f32, b16 = oracle.dequantize(codes, scales, rows, cols, layout, rht, 11)
    assert (f32 == 0).mean() > 0.2
    out = mx.mxfp4_dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), rows, cols,
                              layout, rht, 11, out_dtype=out_dtype)
    got = host(out)
    # scale code 254 overflows the scaled butterfly (Inf - Inf): NaN payloads
    # differ between the device and the host, so NaNs compare by position
    if out_dtype == torch.float32:
        nan = np.isnan(f32)
        assert np.array_equal(np.isnan(got), nan)
        assert np.array_equal(got[~nan].view(np.uint32), f32[~nan].view(np.uint32))
    else:
        nan = np.isnan(synth.bf16_to_f32(b16))
        assert np.array_equal(np.isnan(synth.bf16_to_f32(got)), nan)
        assert np.array_equal(got[~nan], b16[~nan])


@pytest.mark.parametrize("rht", [0, 16, 32])
def test_dequantize_mma_scales(rht):
    """Row dequantize reading GEMM-ready scales, with and without the inverse
    RHT (the RHT path's pipelined loop is its own instantiation per scale
    layout)."""
    rows, cols = 200, 256
    x = synth.normal_bf16((rows, cols), 4)
    q = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_ROW, rht, mx.ROUND_RNE, 3, 0, mx.SCALES_MMA)
    out = mx.mxfp4_dequantize(q.codes, q.scales, rows, cols, mx.LAYOUT_1D_ROW, rht, 3, scale_layout=mx.SCALES_MMA)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW, rht, oracle.ROUND_RNE, 3)[:2]
    _, b16 = oracle.dequantize(codes, scales, rows, cols, oracle.LAYOUT_1D_ROW, rht, 3)
    assert np.array_equal(host(out), b16)


@pytest.mark.parametrize("rht", [0, 32])
@pytest.mark.parametrize("mma", [False, True])
def test_dequantize_column_many_tiles(rht, mma):
    """Column dequantize on more 256 x 64 tiles (720) than resident CTAs, so
    that each CTA walks several tiles through its two-tile prefetch ring."""
    rows, cols = 4096, 2880
    x = synth.normal_bf16((rows, cols), 77)
    sl = mx.SCALES_MMA if mma else mx.SCALES_ROWMAJOR
    q = mx.mxfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_COL, rht, mx.ROUND_RNE, 5, 0, sl)
    out = mx.mxfp4_dequantize(q.codes, q.scales, rows, cols, mx.LAYOUT_1D_COL, rht, 5, scale_layout=sl)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_COL, rht, oracle.ROUND_RNE, 5)[:2]
    assert np.array_equal(host(q.codes), codes)
    _, b16 = oracle.dequantize(codes, scales, rows, cols, oracle.LAYOUT_1D_COL, rht, 5)
    assert np.array_equal(host(out), b16)


def test_invalid_arguments_are_rejected():
    x = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXFP4Error) as e:
        mx.mxfp4_quantize(x[:, :48], mx.LAYOUT_1D_ROW)       # 48 not a multiple of 32
    assert e.value.status == mx.MXFP4_ERR_INVALID_ARG
    with pytest.raises(mx.MXFP4Error) as e:
        mx.mxfp4_quantize(x, mx.LAYOUT_1D_ROW, rht_size=8)
    assert e.value.status == mx.MXFP4_ERR_INVALID_ARG
    with pytest.raises(mx.MXFP4Error) as e:
        mx.mxfp4_quantize(x, mx.LAYOUT_1D_ROW, elem_offset=2)
    assert e.value.status == mx.MXFP4_ERR_INVALID_ARG


@pytest.mark.parametrize("scale_layout", [mx.SCALES_ROWMAJOR, mx.SCALES_MMA])
@pytest.mark.parametrize("rnd", [mx.ROUND_RNE, mx.ROUND_SR])
@pytest.mark.parametrize("rht", [0, 16, 32])
@pytest.mark.parametrize("shape", [(96, 160), (256, 384), (320, 2880)])
def test_dual_row_and_col_bit_exact(shape, rht, rnd, scale_layout):
    rows, cols = shape
    x = synth.student_t_bf16(shape, seed=400 + rows)
    qr, qc = mx.mxfp4_quantize_dual(dev_bf16(x), rht, rnd, 42, scale_layout=scale_layout)
    cr, sr_ = oracle.quantize(x, oracle.LAYOUT_1D_ROW, 0, rnd, 42)
    cc, sc = oracle.quantize(x, oracle.LAYOUT_1D_COL, rht, rnd, 42)
    assert np.array_equal(host(qr.codes), cr) and np.array_equal(host(qc.codes), cc)
    if scale_layout == mx.SCALES_MMA:
        assert np.array_equal(from_mma(host(qr.scales), rows, cols), sr_)
        assert np.array_equal(from_mma(host(qc.scales), cols, rows), sc)
    else:
        assert np.array_equal(host(qr.scales), sr_) and np.array_equal(host(qc.scales), sc)


def test_dual_single_outputs_and_offsets():
    x = synth.student_t_bf16((128, 256), seed=9)
    qr, qc = mx.mxfp4_quantize_dual(dev_bf16(x), 32, mx.ROUND_SR, 5, row_elem_offset=4096, col_elem_offset=8,
                                    col=False)
    assert qc is None
    assert np.array_equal(host(qr.codes), oracle.quantize(x, oracle.LAYOUT_1D_ROW, 0, oracle.ROUND_SR, 5, 4096)[0])
    qr, qc = mx.mxfp4_quantize_dual(dev_bf16(x), 32, mx.ROUND_SR, 5, col_elem_offset=8, row=False)
    assert qr is None
    assert np.array_equal(host(qc.codes), oracle.quantize(x, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_SR, 5, 8)[0])


@pytest.mark.parametrize("scale_layout", [mx.SCALES_ROWMAJOR, mx.SCALES_MMA])
@pytest.mark.parametrize("rnd", [mx.ROUND_RNE, mx.ROUND_SR])
def test_dual_rows_token_slices_equal_the_whole(rnd, scale_layout):
    """Data-parallel token split: each slice quantized with
    mxfp4_quantize_dual_rows equals its part of the whole tensor's dual
    quantization (row blocks: its rows; column blocks along tokens with RHT-32:
    its token columns), bit for bit, SR included; and both equal the oracle
    run on the slice with the whole view's row length."""
    T, C = 384, 320
    x = synth.student_t_bf16((T, C), seed=77)
    xd = dev_bf16(x)
    wr, wc = mx.mxfp4_quantize_dual(xd, 32, rnd, 42)
    wrc, wrs, wcc, wcs = host(wr.codes), host(wr.scales), host(wc.codes), host(wc.scales)
    for t0, n in ((0, 128), (128, 96), (224, 160)):
        qr, qc = mx.mxfp4_quantize_dual_rows(xd[t0:t0 + n], t0, T, 32, rnd, 42, scale_layout=scale_layout)
        assert np.array_equal(host(qr.codes), wrc[t0:t0 + n])
        assert np.array_equal(host(qc.codes), wcc[:, t0 // 2:(t0 + n) // 2])
        sr_, sc = host(qr.scales), host(qc.scales)
        if scale_layout == mx.SCALES_MMA:
            sr_, sc = from_mma(sr_, n, C), from_mma(sc, C, n)
        assert np.array_equal(sr_, wrs[t0:t0 + n]) and np.array_equal(sc, wcs[:, t0 // 32:(t0 + n) // 32])
        part = np.ascontiguousarray(x[t0:t0 + n])
        oc, os_ = oracle.quantize(part, oracle.LAYOUT_1D_COL, 32, rnd, 42, elem_offset=t0, sr_ld=T)
        assert np.array_equal(host(qc.codes), oc) and np.array_equal(sc, os_)


RULES = [(mx.SCALE_ROUNDUP, oracle.SCALE_ROUNDUP), (mx.SCALE_PRESCALE_34, oracle.SCALE_PRESCALE_34)]


@pytest.mark.parametrize("rule", RULES)
@pytest.mark.parametrize("rnd", [mx.ROUND_RNE, mx.ROUND_SR])
@pytest.mark.parametrize("rht", [0, 32])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_scale_rules_bit_exact(layout, rht, rnd, rule):
    rows, cols = SHAPES[layout]
    x = synth.student_t_bf16((rows, cols), seed=500 + layout + rht)
    trans = layout == mx.LAYOUT_2D
    q = mx.mxfp4_quantize(dev_bf16(x), layout, rht, rnd, 42, transposed_copy=trans, scale_rule=rule[0])
    ref = oracle.quantize(x, layout, rht, rnd, 42, transposed_copy=trans, scale_rule=rule[1])
    assert np.array_equal(host(q.codes), ref[0])
    assert np.array_equal(host(q.scales), ref[1])
    if trans:
        assert np.array_equal(host(q.codes_t), ref[2])


@pytest.mark.parametrize("rule", RULES)
def test_scale_rules_every_bf16_pattern(rule):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    a = np.random.default_rng(6).permutation(allbits).reshape(256, 256)
    b = a.copy()
    b[:, ::32] = 0x40C0                                   # 6.0: the round-up boundary
    x = np.concatenate([a, b], axis=0)
    for layout in LAYOUTS:
        for rnd in (mx.ROUND_RNE, mx.ROUND_SR):
            q = mx.mxfp4_quantize(dev_bf16(x), layout, 0, rnd, 9, scale_rule=rule[0])
            ref = oracle.quantize(x, layout, 0, rnd, 9, scale_rule=rule[1])
            assert np.array_equal(host(q.codes), ref[0]), (layout, rnd)
            assert np.array_equal(host(q.scales), ref[1]), (layout, rnd)


@pytest.mark.parametrize("rule", RULES)
def test_scale_rules_dual(rule):
    x = synth.student_t_bf16((256, 384), seed=510)
    qr, qc = mx.mxfp4_quantize_dual(dev_bf16(x), 32, mx.ROUND_SR, 42, scale_rule=rule[0])
    cr, sr_ = oracle.quantize(x, oracle.LAYOUT_1D_ROW, 0, oracle.ROUND_SR, 42, scale_rule=rule[1])
    cc, sc = oracle.quantize(x, oracle.LAYOUT_1D_COL, 32, oracle.ROUND_SR, 42, scale_rule=rule[1])
    assert np.array_equal(host(qr.codes), cr) and np.array_equal(host(qr.scales), sr_)
    assert np.array_equal(host(qc.codes), cc) and np.array_equal(host(qc.scales), sc)


def test_bad_rounding_bits_rejected():
    x = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    for bad in (2, 0x30, 0x40, 0x100):
        with pytest.raises(mx.MXFP4Error) as e:
            mx.mxfp4_quantize(x, mx.LAYOUT_1D_ROW, rounding=bad)
        assert e.value.status == mx.MXFP4_ERR_INVALID_ARG


# ---- NVFP4 ---------------------------------------------------------------------------

@pytest.mark.parametrize("scale_layout", [mx.SCALES_ROWMAJOR, mx.SCALES_MMA])
@pytest.mark.parametrize("rnd", [mx.ROUND_RNE, mx.ROUND_SR])
@pytest.mark.parametrize("layout", [mx.LAYOUT_1D_ROW, mx.LAYOUT_1D_COL])
def test_nvfp4_quantize_bit_exact(layout, rnd, scale_layout):
    rows, cols = (80, 224) if layout == mx.LAYOUT_1D_ROW else (224, 80)
    x = synth.student_t_bf16((rows, cols), seed=600 + layout)
    q = mx.mxfp4_nvfp4_quantize(dev_bf16(x), layout, rnd, 42, scale_layout=scale_layout)
    codes, scales, amax = oracle.nvfp4_quantize(x, layout, rnd, 42)
    assert float(q.amax.item()) == amax
    assert np.array_equal(host(q.codes), codes)
    s = host(q.scales)
    if scale_layout == mx.SCALES_MMA:
        K = q.k
        s = np.array([[s[((r // 128) * ((K // 16 + 3) // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4
                         + kb % 4] for kb in range(scales.shape[1])] for r in range(scales.shape[0])], np.uint8)
    assert np.array_equal(s, scales)


def test_nvfp4_every_bf16_pattern_and_specials():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = allbits[(allbits & 0x7F80) != 0x7F80]                     # no NaN / Inf
    g = np.random.default_rng(8)
    x = g.permutation(np.resize(finite, 256 * 256)).reshape(256, 256)
    for rnd in (mx.ROUND_RNE, mx.ROUND_SR):
        q = mx.mxfp4_nvfp4_quantize(dev_bf16(x), mx.LAYOUT_1D_ROW, rnd, 9)
        codes, scales, amax = oracle.nvfp4_quantize(x, oracle.LAYOUT_1D_ROW, rnd, 9)
        assert np.array_equal(host(q.codes), codes) and np.array_equal(host(q.scales), scales)
    for bad in (0x7FC0, 0xFF80):                                      # NaN, -Inf
        y = x.copy()
        y[5, 9] = bad
        q = mx.mxfp4_nvfp4_quantize(dev_bf16(y), mx.LAYOUT_1D_ROW)
        codes, scales, _ = oracle.nvfp4_quantize(y, oracle.LAYOUT_1D_ROW)
        assert np.array_equal(host(q.codes), codes) and np.array_equal(host(q.scales), scales)
    z = mx.mxfp4_nvfp4_quantize(torch.zeros((32, 64), dtype=torch.bfloat16, device="cuda"))
    assert float(z.amax.item()) == 0.0 and not host(z.codes).any() and not host(z.scales).any()


@pytest.mark.parametrize("k", [-120, -106, -100, -94, 0, 94, 100, 106, 112])
def test_nvfp4_division_at_extreme_scales(k):
    """The element division by the block's X takes an FMA-corrected
    reciprocal when X lies in [2^-100, 2^100] and every nonzero element is at
    least 2^-100, the IEEE division otherwise.  Tensors scaled by 2^k put
    their blocks on both sides of those limits (k = -106 and below: tiny
    elements and divisors; 94 and above: divisors near the top), with a spread
    of block magnitudes and exact zeros; codes and scales must match the
    oracle bit for bit under RNE and SR, in both layouts."""
    rows, cols = 64, 256
    base = synth.student_t_bf16((rows, cols), seed=700 + k)
    f = synth.bf16_to_f32(base).astype(np.float64)
    f *= np.exp2(np.random.default_rng(701).integers(-6, 7, size=(rows, 1)).astype(np.float64))   # row spread
    f[3, :40] = 0.0
    x = synth.bf16_bits((f * 2.0 ** k).astype(np.float32))
    for layout in (mx.LAYOUT_1D_ROW, mx.LAYOUT_1D_COL):
        for rnd in (mx.ROUND_RNE, mx.ROUND_SR):
            q = mx.mxfp4_nvfp4_quantize(dev_bf16(x), layout, rnd, 13)
            codes, scales, _ = oracle.nvfp4_quantize(x, layout, rnd, 13)
            assert np.array_equal(host(q.codes), codes), (layout, rnd)
            assert np.array_equal(host(q.scales), scales), (layout, rnd)


@pytest.mark.parametrize("layout", [mx.LAYOUT_1D_ROW, mx.LAYOUT_1D_COL])
def test_nvfp4_dequantize_matches_oracle(layout):
    rows, cols = 96, 160
    x = synth.student_t_bf16((rows, cols), seed=610)
    q = mx.mxfp4_nvfp4_quantize(dev_bf16(x), layout, mx.ROUND_SR, 3)
    out = host(mx.mxfp4_nvfp4_dequantize(q, rows, cols))
    codes, scales, amax = oracle.nvfp4_quantize(x, layout, oracle.ROUND_SR, 3)
    ref = oracle.nvfp4_dequantize(codes, scales, rows, cols, layout, amax)
    assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))
