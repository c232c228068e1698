"""Oracle pins: the scale-rule variants ("MXFP4", "Clipping in the reference
algorithm" and the "Training with MXFP4" table).

round-up:  the decode scale amax / 6 rounded up to the next power of two, so
           that nothing saturates; in the worst case the +-4 and +-6 codes go
           unused and about 2.58 of FP4's 3.58 binades are used.
3/4 pre-scale: inputs multiplied by 3/4 before quantizing so that no value
           lands in the clipping range (the block exponent still follows the
           unscaled amax).
"""
import math

import numpy as np

import oracle
import synth

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _bf16_positive_finite():
    bits = np.arange(1, 0x7F80, dtype=np.uint32)            # +0 excluded, below +Inf
    return (bits << 16).view(np.float32)


def test_roundup_closed_form_over_every_positive_bf16():
    """Brute force: the smallest integer e with 6 * 2^e >= amax, clamped to the
    E8M0 range, for every positive finite bf16 amax."""
    for amax in _bf16_positive_finite()[::7].tolist() + [6.0, 6.0 * 2 ** 20, 12.0, 3.0, 3.0000002]:
        e = -140
        while 6.0 * 2.0 ** e < amax:
            e += 1
        want = min(max(e + 127, 0), 254)
        assert oracle.scale_code_rule(amax, oracle.SCALE_ROUNDUP) == want, amax


def test_roundup_special_values():
    assert oracle.scale_code_rule(float("nan"), oracle.SCALE_ROUNDUP) == 0xFF
    assert oracle.scale_code_rule(float("inf"), oracle.SCALE_ROUNDUP) == 0xFF
    assert oracle.scale_code_rule(0.0, oracle.SCALE_ROUNDUP) == 0
    # on the boundary amax = 6 * 2^k the scale is 2^k (6 is representable)
    for k in (-3, 0, 5):
        assert oracle.scale_code_rule(6.0 * 2.0 ** k, oracle.SCALE_ROUNDUP) == 127 + k


def _blocks(rows=512, cols=256, seed=21):
    return synth.student_t_bf16((rows, cols), seed=seed)


def test_roundup_never_saturates():
    x = _blocks()
    v = synth.bf16_to_f32(x).astype(np.float64).reshape(-1, 32)
    _, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW, scale_rule=oracle.SCALE_ROUNDUP)
    X = np.ldexp(1.0, scales.reshape(-1).astype(np.int64) - 127)
    assert np.all(np.abs(v).max(axis=1) / X <= 6.0)
    # while the reference rule does push some block maxima past 6
    _, s0 = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    X0 = np.ldexp(1.0, s0.reshape(-1).astype(np.int64) - 127)
    assert np.any(np.abs(v).max(axis=1) / X0 > 6.0)


def test_roundup_worst_case_leaves_4_and_6_unused():
    """A block maximum just above 6 * 2^k scales to just above 3: the codes of
    +-4 and +-6 cannot occur, and the block uses log2(3 / 0.5) = 2.58 of the
    log2(6 / 0.5) = 3.58 binades of the E2M1 grid."""
    vals = np.linspace(-6.0, 6.0, 32).astype(np.float32)
    vals[7] = np.float32(6.03125)                            # the bf16 value just above 6
    x = synth.bf16_bits(vals)[None, :]
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW, scale_rule=oracle.SCALE_ROUNDUP)
    assert oracle.e8m0_decode(int(scales[0, 0])) == 2.0
    nib = np.concatenate([codes[0] & 0xF, codes[0] >> 4])
    assert not np.any(np.isin(nib & 7, [6, 7]))
    top = float(np.abs(synth.bf16_to_f32(x)).max()) / 2.0    # 3.015625
    # binades from the subnormal 0.5 to the block maximum: 2.59 here, tending
    # to log2(3 / 0.5) = 2.585 as the maximum approaches 6 from above; 3.58 in all
    assert 2.585 < math.log2(top / 0.5) < 2.6
    assert round(math.log2(3 / 0.5), 2) == 2.58 and round(math.log2(6 / 0.5), 2) == 3.58


def test_prescale_worked_example():
    """The page's clipping example under the 3/4 pre-scale: amax 7.5 keeps the
    scale 1 and 7.5 is stored as 3/4 of it, 5.625, rounded to 6 -- by rounding,
    not clipping (5.625 < 6)."""
    vals = np.full(32, 0.5, np.float32)
    vals[5] = 7.5
    x = synth.bf16_bits(vals)[None, :]
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW, scale_rule=oracle.SCALE_PRESCALE_34)
    assert oracle.e8m0_decode(int(scales[0, 0])) == 1.0
    assert oracle.e2m1_decode((int(codes[0, 2]) >> 4) & 0xF) == 6.0
    assert oracle.e2m1_decode(int(codes[0, 0]) & 0xF) == 0.5   # 0.375 rounds to 0.5


def test_prescale_removes_clipping():
    """~3% of entries land above 6 under the reference rule; with the 3/4
    pre-scale none does (0.75 * amax / X < 0.75 * 8 = 6)."""
    x = _blocks(seed=22)
    v = synth.bf16_to_f32(x).reshape(-1, 32)
    _, s0 = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    _, s2 = oracle.quantize(x, oracle.LAYOUT_1D_ROW, scale_rule=oracle.SCALE_PRESCALE_34)
    assert np.array_equal(s0, s2)                            # exponent from the unscaled amax
    X = np.ldexp(1.0, s2.reshape(-1, 1).astype(np.int64) - 127)
    pre = (np.float32(0.75) * v).astype(np.float64) / X
    assert np.all(np.abs(pre) < 6.0)
    clipped_ref = np.mean(np.abs(v.astype(np.float64)) / X > 6.0)
    assert clipped_ref > 0.005


def test_prescale_codes_are_rne_of_three_quarters():
    """Each code is the reference conversion of the fp32 value 0.75 * Vi / X."""
    x = _blocks(rows=64, seed=23)
    v = synth.bf16_to_f32(x).reshape(-1, 32)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW, scale_rule=oracle.SCALE_PRESCALE_34)
    e = scales.reshape(-1).astype(np.int64) - 127
    c = codes.reshape(-1, 16)
    nib = np.stack([c & 0xF, c >> 4], axis=-1).reshape(-1, 32)
    for b in range(0, v.shape[0], 7):
        for i in range(32):
            s = np.float32(np.float32(0.75) * v[b, i])
            want = oracle.e2m1_rne(float(np.ldexp(np.float64(s), -int(e[b]))))
            assert int(nib[b, i]) == want
