"""Pins of the oracle's vector search against definitions outside it:

- the estimate of every (query, record) pair equals <q, x_hat> on the
  dequantized record (the packed-code identity the attention pins use),
  evaluated here with plain Python loops on a tiny database;
- the top-k is brute force: Python's sorted() on (-estimate, index);
- k at least N returns every record, in that order;
- equal estimates (duplicated records) come out by index;
- for a well-separated database (the same vectors quantized at 4 bits) the
  nearest neighbour by inner product of the exact vectors is found.
"""

import numpy as np
import pytest

from oracle import quantizer as OQ
from oracle import search as OS


def brute(qz, qs, X):
    enc = OQ.encode(qz, X, aux=False)
    Xh = OQ.dequant(qz, enc)
    out = []
    for q in qs:
        est = [sum(float(q[i]) * float(xh[i]) for i in range(len(q))) for xh in Xh]
        out.append(est)
    return enc, np.array(out)


@pytest.mark.parametrize("variant,bits,rotation", [("mse", 3, "hadamard"), ("prod", 3, "hadamard"),
                                                   ("mse", 2, "dense"), ("prod", 2, "dense")])
def test_scores_and_topk_equal_brute_force(variant, bits, rotation):
    rng = np.random.default_rng(7)
    d, N, nq, k = 16, 40, 3, 7
    X = rng.standard_normal((N, d)).astype(np.float32)
    qs = rng.standard_normal((nq, d)).astype(np.float32)
    qz = OQ.Quantizer(d, bits, variant, seed_rot=3, seed_qjl=4, rotation=rotation)
    enc, est_ref = brute(qz, qs, X)
    est = OS.scores(qz, qs, enc)
    np.testing.assert_allclose(est, est_ref, rtol=1e-9, atol=1e-12)
    vals, idx = OS.topk(est, k)
    for i in range(nq):
        want = sorted(range(N), key=lambda j: (-est[i, j], j))[:k]
        assert list(idx[i]) == want
        np.testing.assert_array_equal(vals[i], est[i, want])


def test_k_beyond_n_and_ties_by_index():
    rng = np.random.default_rng(8)
    d = 32
    X = rng.standard_normal((5, d)).astype(np.float32)
    X = np.concatenate([X, X[2:3], X[2:3]])  # records 5 and 6 duplicate record 2
    q = rng.standard_normal((1, d)).astype(np.float32)
    qz = OQ.Quantizer(d, 4, "mse", seed_rot=1)
    enc = OQ.encode(qz, X, aux=False)
    vals, idx = OS.search_topk(qz, q, enc, 100)
    assert idx.shape == (1, 7)
    assert sorted(idx[0]) == list(range(7))
    pos = {j: p for p, j in enumerate(idx[0])}
    assert pos[2] < pos[5] < pos[6]
    assert np.all(np.diff(vals[0]) <= 0)


def test_nearest_neighbour_of_separated_database_is_found():
    rng = np.random.default_rng(9)
    d, N = 64, 500
    X = rng.standard_normal((N, d)).astype(np.float32)
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    qs = X[[3, 77, 250]] + 0.01 * rng.standard_normal((3, d)).astype(np.float32)
    qz = OQ.Quantizer(d, 4, "mse", seed_rot=2)
    _, idx = OS.search_topk(qz, qs, OQ.encode(qz, X, aux=False), 1)
    assert list(idx[:, 0]) == [3, 77, 250]
