"""Distortion and inner-product bias (oracle side; test infrastructure).

MSE: E ||x - x_hat||^2 for unit x ("The Distortion Guarantee", Theorem 1 and
the measured values it lists for b = 1..4).  Bias: the error of the
inner-product estimate <q, x_hat> against <q, x> ("TurboQuant của Google",
section "Vấn đề của inner product", Fig. 1 and Fig. 2; "内存厂商的噩梦来了",
section 4.2: a 1-bit MSE quantizer scales inner products by about 2/pi).
"""

import numpy as np

from . import quantizer as _qz


def unit_vectors(rng: np.random.Generator, n: int, d: int) -> np.ndarray:
    """Normalised Gaussian rows: uniform on the unit sphere, fp32."""
    x = rng.standard_normal((n, d))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    return x.astype(np.float32)


def mse(qz, x: np.ndarray):
    """(mean, standard error) of ||x - dequant(encode(x))||^2 over the rows."""
    enc = _qz.encode(qz, x)
    xh = _qz.dequant(qz, enc)
    err = np.sum((x.astype(np.float64) - xh) ** 2, axis=1)
    return float(err.mean()), float(err.std(ddof=1) / np.sqrt(len(err)))


def inner_product_errors(qz, x: np.ndarray, q: np.ndarray):
    """(estimate, truth) of <q_i, x_i> for paired rows, estimate through the
    quantizer's reconstruction."""
    enc = _qz.encode(qz, x)
    xh = _qz.dequant(qz, enc)
    est = np.sum(q.astype(np.float64) * xh, axis=1)
    tru = np.sum(q.astype(np.float64) * x.astype(np.float64), axis=1)
    return est, tru


def regression_slope(est: np.ndarray, tru: np.ndarray) -> float:
    """Least-squares slope of est on tru through the origin."""
    return float(np.dot(est, tru) / np.dot(tru, tru))
