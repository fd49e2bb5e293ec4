"""Pins of the oracle's dense (Haar) rotation option against what fixes it
from outside the oracle:

- the defining property of the rotation: Pi is the Q factor of G = Q R with
  R upper triangular with a positive diagonal ("TurboQuant của Google",
  section "Trick đầu tiên": QR of a Gaussian matrix; the positive-diagonal
  choice is what makes Q Haar-distributed), checked by forming Pi^T G;
- orthogonality;
- the Haar law: entries average 0 with second moment 1/d over seeds, the
  diagonal included (a QR without the sign fix has a one-signed diagonal);
  a coordinate of Pi x for a fixed unit x follows the sphere marginal,
  (1 + u) / 2 ~ Beta((d-1)/2, (d-1)/2) (same section);
- a special case that reduces to the separately pinned Hadamard path: the
  dense encoder given the Sylvester matrix H diag(sigma) / sqrt(d) as Pi
  yields the Hadamard encoder's codes (except within rounding of a
  threshold); a transposed Pi would not;
- distortion between the bounds 1/4^b and 2.72/4^b ("The Distortion
  Guarantee", Theorem 1) and equal to the sphere integral, at d = 64 and at
  d = 200, which the Hadamard path cannot take;
- packed-cache attention with dense keys and values equals dense attention on
  the dequantized cache.
"""

import math

import numpy as np
import pytest
from scipy import stats

from oracle import attention as OA
from oracle import codebook as cb
from oracle import metrics as OM
from oracle import prng
from oracle import quantizer as OQ
from oracle import rotation as rot


@pytest.mark.parametrize("d", [8, 64, 200])
def test_haar_matrix_is_the_q_factor_with_positive_r_diagonal(d):
    G = prng.gaussian_matrix_f64(11, d)
    P = rot.haar_matrix(11, d)
    R = P.T @ G
    assert np.abs(np.tril(R, -1)).max() < 1e-10 * np.abs(R).max()
    assert np.all(np.diag(R) > 0)
    assert np.abs(P @ P.T - np.eye(d)).max() < 1e-12
    P32 = P.astype(np.float32).astype(np.float64)
    assert np.abs(P32 @ P32.T - np.eye(d)).max() < 1e-6


def test_haar_law_entries_and_diagonal():
    d, seeds = 8, 400
    Ps = np.stack([rot.haar_matrix(1000 + s, d) for s in range(seeds)])
    for a in (Ps.reshape(seeds, -1), np.einsum("sii->si", Ps)):
        m = a.mean()
        se = a.std(ddof=1) / math.sqrt(a.size)
        assert abs(m) < 4 * se + 1e-12, (m, se)
    sq = (Ps ** 2).reshape(-1)
    assert abs(sq.mean() - 1.0 / d) < 4 * sq.std(ddof=1) / math.sqrt(sq.size)


def test_haar_rotation_of_a_fixed_vector_is_uniform_on_the_sphere():
    d, seeds = 16, 600
    x = np.zeros(d)
    x[3] = 1.0
    u = np.array([(rot.haar_matrix(5000 + s, d) @ x)[0] for s in range(seeds)])
    a = (d - 1) / 2.0
    res = stats.kstest((1.0 + u) / 2.0, stats.beta(a, a).cdf)
    assert res.pvalue > 1e-3, res


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 4])
def test_dense_encoder_with_the_hadamard_matrix_reproduces_hadamard_codes(d, bits):
    rng = np.random.default_rng(d + bits)
    x = rng.standard_normal((3000, d)).astype(np.float32)
    qh = OQ.Quantizer(d, bits, "mse", seed_rot=7)
    qd = OQ.Quantizer(d, bits, "mse", seed_rot=7, rotation="dense")
    qd.Pi = rot.rotation_matrix(qh.signs).astype(np.float32)
    eh, ed = OQ.encode(qh, x), OQ.encode(qd, x)
    np.testing.assert_array_equal(eh["norms"], ed["norms"])
    ih = OQ.unpack_bits(eh["codes"], d, bits)
    idd = OQ.unpack_bits(ed["codes"], d, bits)
    diff = ih != idd
    # the two differ only in rounding (fp32 butterflies vs float64 product)
    gap = np.abs(ed["u"][:, :, None] - qd.thresholds.astype(np.float64)[None, None, :]).min(axis=2)
    assert np.all(gap[diff] < 1e-6)
    assert diff.sum() <= 1e-4 * diff.size
    # a transposed rotation matrix is not the same encoder
    qd.Pi = np.ascontiguousarray(qd.Pi.T)
    assert (OQ.unpack_bits(OQ.encode(qd, x)["codes"], d, bits) != ih).mean() > 0.3


@pytest.mark.parametrize("d", [64, 200])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_dense_distortion_between_bounds_and_equal_to_the_sphere_integral(d, bits):
    rng = np.random.default_rng(100 * d + bits)
    x = OM.unit_vectors(rng, 6000, d)
    qz = OQ.Quantizer(d, bits, "mse", seed_rot=3, rotation="dense")
    mse, se = OM.mse(qz, x)
    assert 1.0 / 4 ** bits < mse < (math.sqrt(3) * math.pi / 2) / 4 ** bits
    _, _, c64, _ = cb.codebook(d, bits)
    want = cb.sphere_distortion(c64, d)
    assert abs(mse - want) < 4 * se, (mse, want, se)


@pytest.mark.parametrize("kvar", ["mse", "prod"])
def test_dense_packed_attention_equals_attention_on_dequantized_cache(kvar):
    d, N, g = 64, 300, 3
    rng = np.random.default_rng(9)
    K = rng.standard_normal((N, d)).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    q = rng.standard_normal((1, g, d)).astype(np.float32)
    kq = OQ.Quantizer(d, 3, kvar, seed_rot=21, seed_qjl=22, rotation="dense")
    vq = OQ.Quantizer(d, 2, "mse", seed_rot=23, rotation="dense")
    ke, ve = OQ.encode(kq, K, aux=False), OQ.encode(vq, V, aux=False)
    kc = {k: v[None, None] for k, v in ke.items()}
    vc = {k: v[None, None] for k, v in ve.items()}
    out = OA.decode_attention(kq, vq, q, kc, vc)
    Kh, Vh = OQ.dequant(kq, ke), OQ.dequant(vq, ve)
    for h in range(g):
        ref = OA.dense_attention(q[0, h], Kh, Vh)
        np.testing.assert_allclose(out[0, h], ref, rtol=1e-9, atol=1e-12)


def test_dense_prod_estimator_is_unbiased_over_qjl_seeds():
    d, pairs, seeds = 64, 256, 48
    rng = np.random.default_rng(4)
    x = OM.unit_vectors(rng, pairs, d)
    q = OM.unit_vectors(rng, pairs, d)
    q = (0.3 * x + math.sqrt(1 - 0.09) * q).astype(np.float32)
    err = []
    for s in range(seeds):
        qz = OQ.Quantizer(d, 2, "prod", seed_rot=100 + s, seed_qjl=200 + s, rotation="dense")
        est, tru = OM.inner_product_errors(qz, x, q)
        err.append(est - tru)
    e = np.concatenate(err)
    assert abs(e.mean()) < 3 * e.std(ddof=1) / math.sqrt(e.size)
