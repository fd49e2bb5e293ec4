"""Pins for the oracle's Lloyd-Max codebooks (CPU).

Each check compares the oracle against something other than itself: the
value a page prints, a closed form, a textbook table, or an independent
numerical integration (scipy.integrate.quad).
"""

import json
import math
import os

import numpy as np
import pytest
from scipy import integrate, special, stats

from oracle import codebook as cb

GOLD = os.path.join(os.path.dirname(__file__), "golden")
PAGES = json.load(open(os.path.join(GOLD, "pages_printed_values.json")))
BOOK = json.load(open(os.path.join(GOLD, "textbook_values.json")))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_one_bit_centroid_is_sqrt_2_over_pi_d(d):
    # the 1-bit Gaussian codebook is +-sqrt(2/(pi d)) (E|Z| for Z ~ N(0,1/d))
    c32, t32, c64, _ = cb.codebook(d, 1)
    want = PAGES["one_bit_centroid_times_sqrt_d"]["value"] / math.sqrt(d)
    assert c64[1] == pytest.approx(want, rel=1e-13)
    assert c64[0] == -c64[1]
    assert abs(float(c32[1]) - want) <= np.spacing(np.float32(want))
    assert t32.tolist() == [0.0]


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_gauss_levels_match_max_1960_table(b):
    c = cb.lloyd_max_gauss(1 << b)
    pos = c[len(c) // 2:]
    np.testing.assert_allclose(pos, BOOK["gauss_lloyd_max_positive_levels"][str(b)], atol=1.5e-4)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_gauss_distortion_matches_table_and_quadrature(b):
    c = cb.lloyd_max_gauss(1 << b)
    closed = cb.gauss_cell_distortion(c)
    assert closed == pytest.approx(BOOK["gauss_lloyd_max_distortion"][str(b)], rel=1e-3)
    t = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    quad = sum(integrate.quad(lambda z, ci=ci: (z - ci) ** 2 * stats.norm.pdf(z), a, bb,
                              epsabs=1e-14)[0] for ci, a, bb in zip(c, t[:-1], t[1:]))
    assert closed == pytest.approx(quad, rel=1e-10)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_gauss_levels_are_a_lloyd_max_fixed_point(b):
    # centroid condition c_i = E[Z | cell i] re-derived by quadrature
    c = cb.lloyd_max_gauss(1 << b)
    t = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    for ci, a, bb in zip(c, t[:-1], t[1:]):
        m1 = integrate.quad(lambda z: z * stats.norm.pdf(z), a, bb, epsabs=1e-15)[0]
        m0 = stats.norm.cdf(bb) - stats.norm.cdf(a)
        assert abs(m1 / m0 - ci) < 1e-12


@pytest.mark.parametrize("d,b", [(64, 2), (128, 3), (128, 4), (256, 4)])
def test_codebook_symmetry_and_thresholds(d, b):
    c32, t32, c64, t64 = cb.codebook(d, b)
    K = 1 << b
    assert np.all(np.diff(c64) > 0)
    np.testing.assert_array_equal(c64, -c64[::-1])
    np.testing.assert_array_equal(c32, -c32[::-1])
    assert t32[K // 2 - 1] == 0.0
    # thresholds are midpoints and separate the centroids
    assert np.all(c32[:-1] < t32) and np.all(t32 < c32[1:])


@pytest.mark.parametrize("d", [64, 128, 256])
def test_beta_one_bit_centroid_closed_form(d):
    # E|X| for a coordinate of a uniform unit vector: Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    c = cb.lloyd_max_beta(2, d)
    want = math.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / math.sqrt(math.pi)
    assert c[1] == pytest.approx(want, rel=1e-12)


def test_beta_levels_fixed_point_by_quadrature():
    d, b = 128, 3
    c = cb.lloyd_max_beta(1 << b, d)
    t = np.concatenate([[-1.0], 0.5 * (c[:-1] + c[1:]), [1.0]])
    f = lambda x: (1 - x * x) ** ((d - 3) / 2)
    for ci, a, bb in zip(c, t[:-1], t[1:]):
        m1 = integrate.quad(lambda x: x * f(x), a, bb, epsabs=1e-17, epsrel=1e-13)[0]
        m0 = integrate.quad(f, a, bb, epsabs=1e-17, epsrel=1e-13)[0]
        assert m1 / m0 == pytest.approx(ci, rel=1e-10)


def test_beta_codebook_tends_to_gauss():
    # the exact coordinate law tends to N(0, 1/d) as d grows
    for d, tol in [(128, 3e-2), (2048, 2e-3)]:
        cbeta = cb.lloyd_max_beta(16, d) * math.sqrt(d)
        cg = cb.lloyd_max_gauss(16)
        np.testing.assert_allclose(cbeta, cg, rtol=tol)


def test_sphere_distortion_reduces_to_gauss_for_large_d():
    c = cb.lloyd_max_gauss(8)
    d = 4096
    assert cb.sphere_distortion(c / math.sqrt(d), d) == pytest.approx(
        cb.gauss_cell_distortion(c), rel=2e-3)
