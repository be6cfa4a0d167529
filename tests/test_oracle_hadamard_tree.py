"""Pins of the oracle's blockwise Hadamard rotation and its reduction tree.

"Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization", 技術概要 §2.2 item 3 (blockwise rotations) and §2.1 (Laplace
data look Gaussian after rotation).
"""
import math

import numpy as np
import pytest
import scipy.linalg
import scipy.stats

NS = [16, 32, 64, 128]


@pytest.mark.parametrize("n", NS)
def test_k_is_nearest_float_to_inv_sqrt(ref, n):
    k = np.float32(ref.hadamard_k(n))
    exact = 1.0 / math.sqrt(n)
    lo, hi = np.nextafter(k, np.float32(0)), np.nextafter(k, np.float32(1))
    assert abs(float(k) - exact) <= abs(float(lo) - exact)
    assert abs(float(k) - exact) <= abs(float(hi) - exact)


@pytest.mark.parametrize("n", NS)
def test_fwht_matrix_is_sylvester_hadamard(ref, n):
    k = np.float32(ref.hadamard_k(n))
    M = ref.fwht(np.eye(n, dtype=np.float32), n)  # row i = FWHT(e_i)
    H = M.astype(np.float64) / float(k)
    assert np.array_equal(H, np.round(H))
    # library routine: scipy's Sylvester-ordered Hadamard matrix
    assert np.array_equal(H, scipy.linalg.hadamard(n).astype(np.float64))
    assert np.array_equal(H @ H.T, n * np.eye(n))


@pytest.mark.parametrize("n", NS)
def test_fwht_small_integers_exact(ref, n):
    rng = np.random.default_rng(n)
    x = rng.integers(-50, 51, size=(64, n)).astype(np.float32)
    y = ref.fwht(x, n)
    Hx = x.astype(np.float64) @ scipy.linalg.hadamard(n).T.astype(np.float64)
    # integer sums are exact in fp32; the only rounding is the multiply by k
    want = (Hx * float(np.float32(ref.hadamard_k(n)))).astype(np.float32)
    assert np.array_equal(y.view(np.uint32), want.view(np.uint32))
    if n in (16, 64):  # k^2 == 1/n exactly: applying it twice is the identity
        assert np.array_equal(ref.fwht(y, n), x)


@pytest.mark.parametrize("n", NS)
def test_fwht_close_to_exact_and_norm_preserving(ref, n):
    rng = np.random.default_rng(100 + n)
    x = rng.standard_normal((256, n)).astype(np.float32)
    y = ref.fwht(x, n).astype(np.float64)
    exact = x.astype(np.float64) @ scipy.linalg.hadamard(n).T / math.sqrt(n)
    # log2(n) rounded add stages plus one rounded multiply, and k itself
    bound = (math.log2(n) + 2) * 2.0 ** -24 * np.abs(x).sum(axis=1, keepdims=True)
    assert np.all(np.abs(y - exact) <= bound)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-5)


def test_fwht_stage_order_is_ascending(ref):
    # Hand-derived: x = [1, 2^-24, 2^-24, 0, ...], n = 16. Ascending stages give
    # after h=1: [1, 1-2^-24, 2^-24, 2^-24] (1 + 2^-24 ties to 1), after h=2:
    # [1, 1, 1-2^-24, 1-2^-23]; the later stages only copy/negate against zeros.
    # A descending order would give [1, 1-2^-24, 1, 1-2^-23] instead.
    e = 2.0 ** -24
    x = np.zeros(16, np.float32)
    x[0], x[1], x[2] = 1.0, e, e
    y = ref.fwht(x, 16)
    want4 = np.array([1.0, 1.0, 1.0 - e, 1.0 - 2 * e], np.float32) * np.float32(0.25)
    assert np.array_equal(y[:4], want4)
    assert np.array_equal(y[4:8], want4) and np.array_equal(y[8:12], want4)


def test_tsum_adjacent_pair_order(ref):
    e = 2.0 ** -24
    # adjacent pairs: (1 + e) -> 1, (0 + e) -> e, 1 + e -> 1
    assert ref.tsum([1.0, e, 0.0, e]) == np.float32(1.0)
    # a strided tree would pair (1, 0) and (e, e) and give 1 + 2^-23
    assert ref.tsum([1.0, e, e, e]) == np.float32(1.0 + 2 * e)
    # left-to-right summation would give 1 here
    rng = np.random.default_rng(3)
    for n in (4, 8, 16, 32, 64, 128):
        v = rng.random(n).astype(np.float32)
        s = float(ref.tsum(v))
        exact = math.fsum(map(float, v))
        assert abs(s - exact) <= math.log2(n) * 2.0 ** -24 * exact
        # parent = left + right exactly (the last level of the tree)
        if n >= 2:
            left, right = ref.tsum(v[: n // 2]), ref.tsum(v[n // 2:])
            assert s == float(np.float32(left) + np.float32(right))


def test_rotation_makes_laplace_gaussian(ref):
    # 技術概要 §2.1: weights/activations look Laplace before and Gaussian after rotation
    rng = np.random.default_rng(5)
    x = rng.laplace(0, 1, size=(2048, 128)).astype(np.float32)
    y = ref.fwht(x, 128)
    kx = scipy.stats.kurtosis(x.ravel(), fisher=False)
    ky = scipy.stats.kurtosis(y.ravel(), fisher=False)
    assert kx > 5.0 and abs(ky - 3.0) < 0.2
