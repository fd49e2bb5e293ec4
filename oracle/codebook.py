"""Lloyd-Max codebooks for the rotated-coordinate distribution (oracle side).

After a random rotation each coordinate of a unit vector follows
f(x) = C (1 - x^2)^((d-3)/2) on [-1, 1], which tends to N(0, 1/d) as d grows
("TurboQuant của Google: nén KV cache 6 lần", section "Trick đầu tiên: xoay
ngẫu nhiên trước khi nén").  The codebook is the 2^b-level scalar quantizer
that minimises the expected squared error against that density, i.e. 1-D
k-means on a continuous density, computed once offline (same page, section
"Lloyd-Max quantizer: chia bucket đúng chỗ"; "The Distortion Guarantee",
section "The Gap": Lloyd-Max applied to a Gaussian).

Readings taken here (the pages give no numerical procedure):
  * default density: N(0, 1/d) ("gauss"); the exact sphere density ("beta")
    is an option;
  * Lloyd's alternation in float64: thresholds are midpoints of adjacent
    centroids, centroids are conditional means of their cell; gauss starts
    from levels equally spaced on [-2, 2] (N(0,1) units) and stops when no
    centroid moves by 1e-15; beta starts from the gauss levels / sqrt(d),
    integrates each cell with 128-node Gauss-Legendre, and stops when no
    centroid moves by 1e-16 (unit-sphere units); both stop after at most
    200000 sweeps;
  * the result is made exactly antisymmetric, c_i = -c_{K-1-i}, the gauss
    levels are divided by sqrt(d), thresholds are the float64 midpoints, and
    both are rounded once to fp32.  For even K the middle threshold is 0.
"""

import math

import numpy as np

_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def _phi(x: float) -> float:
    if math.isinf(x):
        return 0.0
    return _INV_SQRT_2PI * math.exp(-0.5 * x * x)


def _upper_tail(x: float) -> float:
    """P(Z > x) for Z ~ N(0,1)."""
    if x == math.inf:
        return 0.0
    if x == -math.inf:
        return 1.0
    return 0.5 * math.erfc(x / _SQRT2)


def _mass(a: float, b: float) -> float:
    """P(a < Z <= b), written to avoid cancellation in either tail."""
    if a >= 0.0:
        return _upper_tail(a) - _upper_tail(b)
    if b <= 0.0:
        return _upper_tail(-b) - _upper_tail(-a)
    return 1.0 - _upper_tail(b) - _upper_tail(-a)


def lloyd_max_gauss(levels: int, max_sweeps: int = 200000, tol: float = 1e-15):
    """Lloyd-Max centroids of N(0,1) with ``levels`` cells, float64, ascending.

    Centroid of cell (a, b]: E[Z | a < Z <= b] = (phi(a) - phi(b)) / P(a<Z<=b).
    """
    K = levels
    if K == 1:
        return np.zeros(1)
    c = [-2.0 + 4.0 * i / (K - 1) for i in range(K)]
    for _ in range(max_sweeps):
        t = [-math.inf] + [0.5 * (c[i] + c[i + 1]) for i in range(K - 1)] + [math.inf]
        new = []
        for i in range(K):
            a, b = t[i], t[i + 1]
            new.append((_phi(a) - _phi(b)) / _mass(a, b))
        delta = max(abs(new[i] - c[i]) for i in range(K))
        c = new
        if delta < tol:
            break
    c = np.array(c, dtype=np.float64)
    return 0.5 * (c - c[::-1])


def _beta_log_density(x: np.ndarray, d: int) -> np.ndarray:
    return 0.5 * (d - 3) * np.log1p(-x * x)


_GL_CACHE = {}


def _gauss_legendre(nodes: int):
    if nodes not in _GL_CACHE:
        _GL_CACHE[nodes] = np.polynomial.legendre.leggauss(nodes)
    return _GL_CACHE[nodes]


def _beta_cell_moments(a: float, b: float, d: int, nodes: int):
    """(int f, int x f) over [a, b] by Gauss-Legendre, f unnormalised."""
    xg, wg = _gauss_legendre(nodes)
    half = 0.5 * (b - a)
    mid = 0.5 * (b + a)
    x = mid + half * xg
    f = np.exp(_beta_log_density(x, d))
    m0 = half * np.sum(wg * f)
    m1 = half * np.sum(wg * x * f)
    return m0, m1


def lloyd_max_beta(levels: int, d: int, nodes: int = 128, max_sweeps: int = 200000,
                   tol: float = 1e-16):
    """Lloyd-Max centroids of the exact coordinate density of a uniform unit
    vector in R^d, float64, ascending, in unit-sphere units."""
    K = levels
    if K == 1:
        return np.zeros(1)
    c = list(lloyd_max_gauss(K) / math.sqrt(d))
    for _ in range(max_sweeps):
        t = [-1.0] + [0.5 * (c[i] + c[i + 1]) for i in range(K - 1)] + [1.0]
        new = []
        for i in range(K):
            m0, m1 = _beta_cell_moments(t[i], t[i + 1], d, nodes)
            new.append(m1 / m0)
        delta = max(abs(new[i] - c[i]) for i in range(K))
        c = new
        if delta < tol:
            break
    c = np.array(c, dtype=np.float64)
    return 0.5 * (c - c[::-1])


def codebook(d: int, bits: int, dist: str = "gauss"):
    """fp32 centroids (2^bits) and thresholds (2^bits - 1) for dimension d.

    ``bits`` is the number of MSE bits b_m; bits == 0 gives the empty codebook
    (TurboQuant_prod at b = 1 keeps only the QJL sketch).
    Returns (centroids_f32, thresholds_f32, centroids_f64, thresholds_f64).
    """
    if bits == 0:
        e = np.zeros(0)
        return e.astype(np.float32), e.astype(np.float32), e, e
    K = 1 << bits
    if dist == "gauss":
        c64 = lloyd_max_gauss(K) / math.sqrt(d)
    elif dist == "beta":
        c64 = lloyd_max_beta(K, d)
    else:
        raise ValueError(dist)
    t64 = 0.5 * (c64[:-1] + c64[1:])
    return c64.astype(np.float32), t64.astype(np.float32), c64, t64


def gauss_cell_distortion(c: np.ndarray) -> float:
    """E[(Z - Q(Z))^2] for Z ~ N(0,1) under nearest-centroid Q with levels c
    (N(0,1) units), in closed form per cell:
    int_a^b (z-c)^2 phi = P - (b phi(b) - a phi(a)) - 2c (phi(a) - phi(b)) + c^2 P.
    """
    K = len(c)
    t = [-math.inf] + [0.5 * (c[i] + c[i + 1]) for i in range(K - 1)] + [math.inf]
    tot = 0.0
    for i in range(K):
        a, b = t[i], t[i + 1]
        P = _mass(a, b)
        bpb = 0.0 if math.isinf(b) else b * _phi(b)
        apa = 0.0 if math.isinf(a) else a * _phi(a)
        i2 = P - (bpb - apa)
        i1 = _phi(a) - _phi(b)
        tot += i2 - 2.0 * c[i] * i1 + c[i] * c[i] * P
    return tot


def sphere_distortion(c: np.ndarray, d: int, nodes: int = 400) -> float:
    """d * E[(X - Q(X))^2] for X a coordinate of a uniform unit vector in R^d
    (the exact per-vector MSE of a scalar quantizer with levels ``c``,
    unit-sphere units), by Gauss-Legendre on each cell of the Beta density."""
    K = len(c)
    t = [-1.0] + [0.5 * (c[i] + c[i + 1]) for i in range(K - 1)] + [1.0]
    xg, wg = _gauss_legendre(nodes)
    num = 0.0
    den = 0.0
    for i in range(K):
        a, b = t[i], t[i + 1]
        half = 0.5 * (b - a)
        x = 0.5 * (a + b) + half * xg
        f = np.exp(_beta_log_density(x, d))
        den += half * np.sum(wg * f)
        num += half * np.sum(wg * f * (x - c[i]) ** 2)
    return d * num / den
