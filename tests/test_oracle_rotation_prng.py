"""Pins for the oracle's rotation and its seeded parameters (CPU)."""

import json
import math
import os

import numpy as np
import pytest
from scipy import stats

from oracle import prng, rotation

GOLD = os.path.join(os.path.dirname(__file__), "golden")
BOOK = json.load(open(os.path.join(GOLD, "textbook_values.json")))


def sylvester(d):
    """Sylvester construction by the Kronecker recursion [[H, H], [H, -H]]
    (independent of the popcount formula the oracle uses)."""
    H = np.array([[1.0]])
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def test_splitmix64_reference_vector():
    got = [prng.splitmix64(1234567, k) for k in range(5)]
    assert got == BOOK["splitmix64_seed_1234567_first5"]


def test_fwht_worked_example():
    # H_4 (1,2,3,4) = (10, -2, -4, 0) by hand
    y = rotation.fwht_f32(np.array([[1, 2, 3, 4]], np.float32))
    assert y.tolist() == [[10.0, -2.0, -4.0, 0.0]]


@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_hadamard_matches_sylvester_and_fwht(d):
    H = rotation.hadamard(d)
    np.testing.assert_array_equal(H, sylvester(d))
    rng = np.random.default_rng(d)
    x = rng.standard_normal((5, d))
    np.testing.assert_allclose(rotation.fwht_f64(x), x @ sylvester(d).T, rtol=0, atol=1e-12)
    y32 = rotation.fwht_f32(x.astype(np.float32)).astype(np.float64)
    exact = x.astype(np.float32).astype(np.float64) @ sylvester(d).T
    # fp32 error bound for log2(d) stages of +-: |err| <= log2 d * u * sum|x|
    bound = math.log2(d) * 2.0 ** -24 * np.abs(x).sum(axis=1, keepdims=True) * 1.01
    assert np.all(np.abs(y32 - exact) <= bound)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rotation_is_orthogonal_and_inverse(d):
    sig = prng.signs(7, d)
    P = rotation.rotation_matrix(sig)
    np.testing.assert_allclose(P @ P.T, np.eye(d), atol=1e-12)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, d))
    y = rotation.rotate_f64(x, sig)
    np.testing.assert_allclose(y, x @ P.T, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(rotation.unrotate_f64(y, sig), x, atol=1e-12)


def test_signs_are_rademacher():
    s = prng.signs(0, 4096)
    assert set(np.unique(s).tolist()) == {-1, 1}
    assert abs(int(s.sum())) < 4 * math.sqrt(4096)
    assert not np.array_equal(prng.signs(0, 128), prng.signs(1, 128))


def test_gaussian_matrix_is_standard_normal():
    S = prng.gaussian_matrix(3, 128).astype(np.float64).ravel()
    assert abs(S.mean()) < 4 / math.sqrt(S.size)
    assert abs(S.var() - 1) < 4 * math.sqrt(2 / S.size)
    assert stats.kstest(S, "norm").pvalue > 1e-3
    # consecutive (cos, sin) pairs are uncorrelated
    assert abs(np.corrcoef(S[0::2], S[1::2])[0, 1]) < 4 / math.sqrt(S.size / 2)


def test_fact1_gaussian_norm_concentrates_near_sqrt_d():
    # "I Spent 31 Hours On The Math Behind Turboquant", property 2: the norm of
    # a standard Gaussian vector concentrates around sqrt(d)
    rng = np.random.default_rng(0)
    for d in (16, 128, 512):
        r = np.linalg.norm(rng.standard_normal((10000, d)), axis=1)
        assert r.mean() == pytest.approx(math.sqrt(d), rel=0.05)
        assert r.std() < 0.75


def test_fact2_projection_is_gaussian_with_norm_variance():
    # property 1 of the same page, restated on a synthetic vector: S x ~ N(0, ||x||^2 I)
    rng = np.random.default_rng(5)
    x = rng.standard_normal(64) * 1.3
    y = np.stack([prng.gaussian_matrix(s, 64)[0] @ x for s in range(400)])
    nx = np.linalg.norm(x)
    assert stats.kstest(y / nx, "norm").pvalue > 1e-3
