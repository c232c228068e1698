"""Oracle pins: the randomized Hadamard transform.

"MXFP4" (aiwiki.ai), "Training with MXFP4": a random Hadamard transform bounds
the variance from block outliers; Hadamard size 32 is used for MXFP4.  The
oracle applies c_d * H_d * diag(s) with H_d the Sylvester Hadamard matrix as an
fp32 butterfly (reading R2).  Pins: the Sylvester closed form
H[i][j] = (-1)^popcount(i & j), H H^T = d I in exact integers, agreement with
an fp64 matrix product within the butterfly's rounding bound, and the inverse
round trip.
"""
import numpy as np
import pytest

import oracle

U = 2.0 ** -24


def _popcount(v):
    return bin(v).count("1")


@pytest.mark.parametrize("d", [16, 32])
def test_butterfly_is_sylvester_hadamard(d):
    H = np.zeros((d, d))
    for j in range(d):
        e = np.zeros(d, np.float32)
        e[j] = 1
        H[:, j] = oracle.fwht_f32(e)
    closed = np.array([[(-1) ** _popcount(i & j) for j in range(d)] for i in range(d)])
    assert np.array_equal(H, closed)
    assert np.array_equal(H.astype(np.int64) @ H.T.astype(np.int64), d * np.eye(d, dtype=np.int64))


def test_normalisation_constants():
    y = oracle.rht_forward(np.eye(1, 32, 0, dtype=np.float32)[0], 0)
    assert np.all(np.abs(y) == y[0])
    assert y.view(np.uint32)[0] == 0x3E3504F3          # fp32(1/sqrt(32))
    y16 = oracle.rht_forward(np.eye(1, 16, 0, dtype=np.float32)[0], 0)
    assert np.all(np.abs(y16) == 0.25)


def _reference(x, d, mask):
    H = np.array([[(-1.0) ** _popcount(i & j) for j in range(d)] for i in range(d)])
    s = np.array([-1.0 if (mask >> j) & 1 else 1.0 for j in range(d)])
    return (H @ (s * x.astype(np.float64))) / np.sqrt(d)


@pytest.mark.parametrize("d", [16, 32])
def test_forward_matches_fp64_matrix_product_within_bound(d):
    g = np.random.default_rng(d)
    L = int(np.log2(d))
    for trial in range(400):
        mask = int(g.integers(0, 2 ** 32))
        scale = 10.0 ** g.uniform(-20, 20)
        x = (g.standard_t(3, d) * scale).astype(np.float32)
        y = oracle.rht_forward(x, mask).astype(np.float64)
        ref = _reference(x, d, mask)
        sabs = np.abs(x.astype(np.float64)).sum()
        bound = (L + 2) * U * sabs / np.sqrt(d) + 2 * U * np.abs(ref)
        assert np.all(np.abs(y - ref) <= bound), (trial, np.max(np.abs(y - ref) - bound))


@pytest.mark.parametrize("d", [16, 32])
def test_inverse_round_trip(d):
    g = np.random.default_rng(100 + d)
    L = int(np.log2(d))
    for trial in range(400):
        mask = int(g.integers(0, 2 ** 32))
        x = (g.standard_normal(d) * 10.0 ** g.uniform(-10, 10)).astype(np.float32)
        back = oracle.rht_inverse(oracle.rht_forward(x, mask), mask).astype(np.float64)
        bound = 2 * (L + 2) * U * d * np.max(np.abs(x))
        assert np.max(np.abs(back - x)) <= bound


def test_sign_mask_flips_the_right_inputs():
    # with a single input set, the output is +-c * H[:, j] * s_j
    d = 32
    mask = 0b1010_0000_0000_0000_0000_0000_0000_0110
    for j in range(d):
        e = np.zeros(d, np.float32)
        e[j] = 1
        y = oracle.rht_forward(e, mask)
        sj = -1 if (mask >> j) & 1 else 1
        expect = np.array([sj * (-1) ** _popcount(i & j) for i in range(d)], np.float64) / np.sqrt(32)
        assert np.allclose(y, expect, rtol=1e-7, atol=0)
