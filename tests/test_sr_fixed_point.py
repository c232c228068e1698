"""The stochastic-rounding decision of the GPU kernels, restated in integer
Python and checked against the definition on exact rationals.

Definition ("MXFP4" (aiwiki.ai), "Conversion rules", with the stochastic
rounding of the ALTO recipe): for a scaled magnitude |v| <= 6 between grid
neighbours lo <= |v| < hi, the code rounds up iff r < f * 2^32 with
f = (|v| - lo) / (hi - lo) and r the element's 32-bit random word.

Kernel form (e2m1_sr_fixed / e2m1x8_sr_tiny in csrc/common.cuh): with ab the
fp32 bits of |v|, e = ab >> 23, s = min(e - 117, 10), m the 24-bit
significand and W = max(ab - 0x3F000000, m), the code is the high word of
W * 2^s + ~r when s >= 0; below 2^-10 (s < 0) it is [r < ceil(m * 2^(e-117))].
These tests pin that identity on CPU; the GPU tests pin the kernels to the
oracle bit for bit.
"""
import math
import random
from fractions import Fraction as F

M32 = 0xFFFFFFFF
SIX = 0x40C00000
GRID = [F(0), F(1, 2), F(1), F(3, 2), F(2), F(3), F(4), F(6)]


def value(ab: int) -> F:
    e, mant = ab >> 23, ab & 0x7FFFFF
    if e == 0:
        return F(mant, 2 ** 149)
    return F(0x800000 | mant, 2 ** (150 - e))


def by_definition(ab: int, r: int) -> int:
    y = value(ab)
    if y >= 6:
        return 7
    i = max(k for k in range(8) if GRID[k] <= y)
    f = (y - GRID[i]) / (GRID[i + 1] - GRID[i])
    return i + (1 if r < f * 2 ** 32 else 0)


def kernel_form(ab: int, r: int) -> int:
    e = ab >> 23
    s = min(e - 117, 10)
    m = (ab & 0x7FFFFF) | 0x800000
    if s < 0:
        if ab == 0:
            return 0
        sh = 117 - e
        t = (((m - 1) >> sh) if sh < 32 else 0) + 1
        return 1 if r < t else 0
    w = max(ab - 0x3F000000, m)
    return ((w << s) + (~r & M32)) >> 32


def _cases():
    rnd = random.Random(2024)
    abs_ = [0, 1, 0x7FFFFF, SIX, 0x3F000000, 0x3F800000, 0x40000000, 0x40800000, 0x3A800000, 0x3A7FFFFF]
    for e in range(0, 130):
        for mant in (0, 1, 0x3FFFFF, 0x400000, 0x7FFFFF):
            abs_.append((e << 23) | mant)
        for _ in range(12):
            abs_.append((e << 23) | rnd.randrange(1 << 23))
    for ab in abs_:
        if ab > SIX:
            continue
        y = value(ab)
        rs = {0, M32, 1 << 23, (1 << 23) - 1, 1 << 31}
        rs.update(rnd.randrange(1 << 32) for _ in range(6))
        if y < 6:
            i = max(k for k in range(8) if GRID[k] <= y)
            t = (y - GRID[i]) / (GRID[i + 1] - GRID[i]) * 2 ** 32
            for base in (math.floor(t), math.ceil(t)):
                for d in (-1, 0, 1):
                    if 0 <= base + d <= M32:
                        rs.add(base + d)
        for r in rs:
            yield ab, r


def test_fixed_point_decision_equals_definition():
    n = 0
    for ab, r in _cases():
        assert kernel_form(ab, r) == by_definition(ab, r), (hex(ab), r)
        n += 1
    assert n > 10000


def test_definition_sanity():
    # on-grid values never move; 6 saturates; the midpoint of [1, 1.5] rounds up iff r < 2^31
    one, one_half, one_quarter = 0x3F800000, 0x3FC00000, 0x3FA00000
    assert by_definition(one, 0) == 2 and by_definition(one_half, 0) == 3
    assert by_definition(SIX, 0) == 7
    assert by_definition(one_quarter, (1 << 31) - 1) == 3 and by_definition(one_quarter, 1 << 31) == 2
