"""Oracle pins: number formats, scale rule, element rounding.

Pinned to what the page "MXFP4" (aiwiki.ai) prints ("Format specification"
tables, "Conversion rules", the worked example in "Clipping in the reference
algorithm") and to closed forms / brute force written independently of the
oracle's own code.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import read_golden


# ---- E2M1 / E8M0 decode -------------------------------------------------------------

def test_e2m1_all_16_codes_match_page_table():
    table = read_golden("e2m1_table.txt")
    assert len(table) == 8
    for bits, value, _kind in table:
        code = int(bits, 2)
        assert oracle.e2m1_decode(code) == float(value)
        # "The negative values have the same pattern with the sign bit set."
        neg = oracle.e2m1_decode(code | 8)
        assert neg == -float(value) and math.copysign(1.0, neg) == -1.0


def test_e2m1_grid_matches_format_parameters():
    p = {k: v for k, v in read_golden("mxfp4_parameters.txt")}
    mags = sorted({abs(oracle.e2m1_decode(c)) for c in range(16)})
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert max(mags) == float(p["element_max_normal"])
    assert min(m for m in mags if m >= 1.0) == float(p["element_min_normal"])
    assert min(m for m in mags if m > 0) == float(p["element_subnormal"])
    # E2M1 with bias 1: normal = 2^(E-1) * (1 + M/2), subnormal = 2^0 * M/2.
    for code in range(8):
        e, m = code >> 1, code & 1
        closed = (2.0 ** (e - 1)) * (1 + m / 2) if e else m / 2
        assert oracle.e2m1_decode(code) == closed


def test_e8m0_all_256_codes():
    p = {k: v for k, v in read_golden("mxfp4_parameters.txt")}
    bias = int(p["scale_bias"])
    nan_code = int(p["scale_nan_code"], 16)
    for code in range(256):
        v = oracle.e8m0_decode(code)
        if code == nan_code:
            assert math.isnan(v)
        else:
            assert v == math.ldexp(1.0, code - bias)
            assert int(p["scale_min_exponent"]) <= code - bias <= int(p["scale_max_exponent"])
    # no zero and no infinity among the codes
    vals = [oracle.e8m0_decode(c) for c in range(255)]
    assert all(v > 0 and math.isfinite(v) for v in vals)


def test_storage_is_136_bits_per_block():
    p = {k: v for k, v in read_golden("mxfp4_parameters.txt")}
    k = int(p["block_size"])
    x = np.zeros((3, 4 * k), np.uint16)
    codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
    bits = (codes.nbytes + scales.nbytes) * 8
    nblocks = x.size // k
    assert bits == nblocks * int(p["bits_per_block"])
    assert bits / x.size == float(p["bits_per_value"])


# ---- scale rule -----------------------------------------------------------------------

def _all_positive_finite_bf16():
    bits = np.arange(1, 0x7F80, dtype=np.uint32)  # +subnormals .. +max finite
    return (bits << 16).view(np.float32)


def test_scale_rule_closed_form_over_every_positive_bf16():
    """X = (largest power of two not above amax) / 4, from exact rational arithmetic."""
    for a in _all_positive_finite_bf16():
        code = oracle.scale_code(float(a))
        fa = Fraction(float(a))
        # exact floor(log2 amax)
        fl = fa.numerator.bit_length() - fa.denominator.bit_length()
        if Fraction(2) ** fl > fa:
            fl -= 1
        assert Fraction(2) ** fl <= fa < Fraction(2) ** (fl + 1)
        e = fl - 2
        expect = min(max(e + 127, 0), 254)
        assert code == expect, (float(a), code, expect)
        if e + 127 >= 0:
            X = Fraction(2) ** (code - 127)
            assert 4 * X <= fa < 8 * X   # block max lands in [4, 8) after scaling


def test_scale_rule_special_cases():
    assert oracle.scale_code(0.0) == 0                   # reading R4
    assert oracle.scale_code(float("nan")) == 0xFF       # reading R3
    assert oracle.scale_code(float("inf")) == 0xFF
    assert oracle.scale_code(6.0) == 127                 # 2^2 <= 6 < 2^3 -> e = 0
    assert oracle.scale_code(8.0) == 128                 # e = 1
    assert oracle.scale_code(4.0) == 127
    assert oracle.scale_code(3.999) == 126
    tiny = float(np.float32(2.0) ** -149)                # smallest fp32 subnormal
    assert oracle.scale_code(tiny) == 0                  # clamped at -127
    assert oracle.scale_code(2.0 ** -125) == 0           # e = -127 exactly
    assert oracle.scale_code(2.0 ** -124) == 1


def test_worked_clipping_example_from_page():
    for amax, scale, stored in read_golden("clipping_example.txt"):
        amax, scale, stored = float(amax), float(scale), float(stored)
        code = oracle.scale_code(amax)
        assert oracle.e8m0_decode(code) == scale
        # whole block through the quantizer: the amax element is stored as 6.
        # The scale follows max |Vi| ("Conversion rules"), so the same holds
        # with the sign flipped: -7.5 is stored as -6 under the same scale.
        for sign in (1.0, -1.0):
            vals = np.full(32, 0.5, np.float32)
            vals[5] = sign * amax
            x = (vals.view(np.uint32) >> 16).astype(np.uint16)[None, :]
            codes, scales = oracle.quantize(x, oracle.LAYOUT_1D_ROW)
            assert oracle.e8m0_decode(int(scales[0, 0])) == scale
            nib = (int(codes[0, 5 // 2]) >> (4 * (5 % 2))) & 0xF
            assert oracle.e2m1_decode(nib) * scale == sign * stored


# ---- element rounding -------------------------------------------------------------------

def _rne_piecewise(v: float) -> float:
    """Round-half-even on each uniformly spaced stretch of the E2M1 grid, using
    Python's round() (which rounds halves to even): spacing 0.5 on [0, 2),
    1 on [2, 4), 2 on [4, 6]; saturate at 6.  On each stretch the parity of the
    stretch index equals the parity of the E2M1 code, so this is ties-to-even."""
    a = abs(v)
    if a >= 6.0:
        return 6.0
    if a < 2.0:
        return min(round(a * 2) / 2, 2.0)
    if a < 4.0:
        return float(min(round(a), 4))
    return float(min(2 * round(a / 2), 6))


def test_rne_tie_table():
    for v, expect in read_golden("rne_ties.txt"):
        v, expect = float(v), float(expect)
        for s in (1.0, -1.0):
            code = oracle.e2m1_rne(s * v)
            assert abs(oracle.e2m1_decode(code)) == expect
            assert (code >> 3) == (1 if s < 0 else 0)


def test_rne_against_piecewise_round_half_even():
    g = np.random.default_rng(123)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    mids = (grid[1:] + grid[:-1]) / 2
    pts = [np.float32(v) for v in np.concatenate([grid, mids, [6.5, 7, 8, 100, 1e30]])]
    near = []
    for p in pts:
        near += [np.nextafter(p, np.float32(0)), np.nextafter(p, np.float32(1e38))]
    rnd = g.uniform(0, 8, 200000).astype(np.float32)
    small = np.float32(2.0) ** g.uniform(-149, 1, 20000).astype(np.float32)
    vals = np.concatenate([np.array(pts + near, np.float32), rnd, small])
    for v in vals:
        for s in (1, -1):
            x = float(np.float32(s * v))
            code = oracle.e2m1_rne(x)
            assert abs(oracle.e2m1_decode(code)) == _rne_piecewise(x), x
            assert (code >> 3) == (1 if math.copysign(1, x) < 0 else 0)


def test_rne_saturates_and_is_nearest():
    for v in [6.0, 6.0001, 7.99, 8.0, 1e6, 3.4e38, float("inf")]:
        assert oracle.e2m1_rne(v) == 7 and oracle.e2m1_rne(-v) == 15
    g = np.random.default_rng(7)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for v in g.uniform(0, 6, 5000).astype(np.float32):
        q = abs(oracle.e2m1_decode(oracle.e2m1_rne(float(v))))
        assert abs(q - v) == np.min(np.abs(grid - v))


def test_negative_zero_code():
    # reading R7: sign preserved, -0 -> code 8
    assert oracle.e2m1_rne(-0.0) == 8
    assert oracle.e2m1_rne(-0.2) == 8
    assert oracle.e2m1_rne(0.2) == 0
