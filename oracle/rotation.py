"""Randomized Hadamard rotation (oracle side; test infrastructure).

The rotation multiplies by a random orthogonal matrix so that every coordinate
of the rotated unit vector has the same known law ("TurboQuant của Google:
nén KV cache 6 lần", section "Trick đầu tiên"; "内存厂商的噩梦来了", section
4.1, step 1).  Its efficient replacement for the dense d x d product is a
Walsh-Hadamard transform ("内存厂商的噩梦来了", the note after the section-4
pseudocode).

Reading taken here: one round, Pi = H D / sqrt(d), with H the Sylvester
Hadamard matrix H[i][j] = (-1)^popcount(i & j) and D = diag(sigma) the seeded
signs; Pi^T = D H / sqrt(d).

``fwht_f32`` is the canonical fp32 transform every encoder must reproduce bit
for bit: stages h = d/2, d/4, ..., 1; at each stage every pair (i, i+h) with
bit h of i clear becomes (fl(a+b), fl(a-b)); no normalisation.

The dense option is the rotation the pages define first ("TurboQuant của
Google", section "Trick đầu tiên": Pi is the Q factor of the QR decomposition
of a matrix of i.i.d. Gaussians), whose d x d product per vector the
critique of the runtime cost names ("Steel-man: ReturningTarzan của ExLlama
đã đúng ở đâu", point 1).  Reading taken here: G is the seeded float64
Gaussian matrix of oracle.prng (row-major); G = Q R with the signs of Q's
columns chosen so that R has a positive diagonal (the choice that makes Q
Haar-distributed: Mezzadri, "How to generate random matrices from the
classical compact groups", 2007); Pi = Q, so y = Pi x; the stored parameter
is Pi rounded once to fp32.  It needs no power-of-two d.
"""

import numpy as np

from . import prng as _prng


def hadamard(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix, float64, entries +-1, built from its
    definition H[i][j] = (-1)^popcount(i & j)."""
    i = np.arange(d)
    pc = np.zeros((d, d), dtype=np.int64)
    x = i[:, None] & i[None, :]
    while np.any(x):
        pc += x & 1
        x >>= 1
    return np.where(pc % 2 == 0, 1.0, -1.0)


def rotation_matrix(sig: np.ndarray) -> np.ndarray:
    """Pi = H diag(sigma) / sqrt(d) in float64."""
    d = sig.shape[0]
    return hadamard(d) * sig.astype(np.float64)[None, :] / np.sqrt(d)


def fwht_f32(y: np.ndarray) -> np.ndarray:
    """Canonical unnormalised FWHT of the rows of ``y`` in fp32 (see module
    docstring for the stage order).  ``y``: [n, d] float32."""
    assert y.dtype == np.float32
    n, d = y.shape
    a = y.copy()
    h = d // 2
    while h >= 1:
        v = a.reshape(n, d // (2 * h), 2, h)
        lo = v[:, :, 0, :]
        hi = v[:, :, 1, :]
        s = lo + hi
        t = lo - hi
        a = np.stack([s, t], axis=2).reshape(n, d)
        h //= 2
    return a


def fwht_f64(y: np.ndarray) -> np.ndarray:
    """Unnormalised FWHT of the rows of ``y`` in float64 (same butterflies)."""
    y = np.asarray(y, dtype=np.float64)
    shape = y.shape
    d = shape[-1]
    a = y.reshape(-1, d).copy()
    n = a.shape[0]
    h = d // 2
    while h >= 1:
        v = a.reshape(n, d // (2 * h), 2, h)
        lo = v[:, :, 0, :]
        hi = v[:, :, 1, :]
        a = np.stack([lo + hi, lo - hi], axis=2).reshape(n, d)
        h //= 2
    return a.reshape(shape)


def rotate_f64(x: np.ndarray, sig: np.ndarray) -> np.ndarray:
    """Pi x = H (sigma * x) / sqrt(d), float64, over the last axis."""
    d = sig.shape[0]
    return fwht_f64(np.asarray(x, np.float64) * sig.astype(np.float64)) / np.sqrt(d)


def unrotate_f64(y: np.ndarray, sig: np.ndarray) -> np.ndarray:
    """Pi^T y = sigma * (H y) / sqrt(d), float64, over the last axis."""
    d = sig.shape[0]
    return sig.astype(np.float64) * fwht_f64(y) / np.sqrt(d)


def haar_matrix(seed: int, d: int) -> np.ndarray:
    """Dense random rotation Pi = Q (float64, d x d) from G = Q R, R with a
    positive diagonal; numpy's QR (LAPACK Householder) is the library step."""
    G = _prng.gaussian_matrix_f64(seed, d)
    Q, R = np.linalg.qr(G)
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s[None, :]
