"""The oracle's pins catch plausible mistakes (CPU).

Each case plants one mistake in the oracle (through monkeypatch, on the CPU)
and checks that a pin which passes for the real oracle fails for the mutant:
a dropped term, a wrong sign, a transposed operand, a missing scale, a
skipped butterfly stage.
"""

import math

import numpy as np
import pytest

from oracle import attention as OA
from oracle import codebook as cb
from oracle import metrics
from oracle import quantizer as Q
from oracle import rotation as R


def sylvester(d):
    H = np.array([[1.0]])
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def fwht_pin_holds():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 64))
    return np.allclose(R.fwht_f64(x), x @ sylvester(64).T, atol=1e-10)


def mse_pin_holds(b=2, d=128):
    rng = np.random.default_rng(1)
    x = metrics.unit_vectors(rng, 2048, d)
    m, se = metrics.mse(Q.Quantizer(d, b), x)
    exact = cb.sphere_distortion(cb.codebook(d, b)[0].astype(np.float64), d)
    return abs(m - exact) < 4 * se and 1 / 4 ** b < m < 2.72 / 4 ** b


def prod_unbiased_pin_holds(b=2, d=128):
    errs = []
    for seed in range(8):
        rng = np.random.default_rng(50 + seed)
        x = metrics.unit_vectors(rng, 1024, d).astype(np.float64)
        z = rng.standard_normal(x.shape)
        z -= np.sum(z * x, axis=1, keepdims=True) * x
        z /= np.linalg.norm(z, axis=1, keepdims=True)
        q = 0.5 * x + math.sqrt(0.75) * z
        qz = Q.Quantizer(d, b, "prod", seed_rot=seed, seed_qjl=100 + seed)
        est, tru = metrics.inner_product_errors(qz, x.astype(np.float32), q)
        errs.append(est - tru)
    e = np.concatenate(errs)
    return abs(e.mean()) < 4 * e.std() / math.sqrt(e.size)


def attention_definition_pin_holds():
    rng = np.random.default_rng(2)
    q, K, V = rng.standard_normal(8), rng.standard_normal((5, 8)), rng.standard_normal((5, 8))
    logits = [sum(a * b for a, b in zip(q, k)) / math.sqrt(8) for k in K]
    m = max(logits)
    e = [math.exp(l - m) for l in logits]
    want = [sum(e[j] / sum(e) * V[j][i] for j in range(5)) for i in range(8)]
    return np.allclose(OA.dense_attention(q, K, V), want, rtol=1e-10)


def test_real_oracle_passes_every_pin():
    assert fwht_pin_holds()
    assert mse_pin_holds()
    assert prod_unbiased_pin_holds()
    assert attention_definition_pin_holds()


def test_skipped_butterfly_stage_is_caught(monkeypatch):
    real = R.fwht_f64

    def mutant(y):
        y = np.asarray(y, np.float64)
        d = y.shape[-1]
        a = y.reshape(-1, d).copy()
        h = d // 2
        while h >= 2:  # stage h = 1 forgotten
            v = a.reshape(a.shape[0], d // (2 * h), 2, h)
            a = np.stack([v[:, :, 0] + v[:, :, 1], v[:, :, 0] - v[:, :, 1]], axis=2).reshape(-1, d)
            h //= 2
        return a.reshape(y.shape)

    monkeypatch.setattr(R, "fwht_f64", mutant)
    assert not fwht_pin_holds()
    monkeypatch.setattr(R, "fwht_f64", real)
    assert fwht_pin_holds()


def test_transposed_rotation_in_dequant_is_caught(monkeypatch):
    # reconstructing with Pi instead of Pi^T
    monkeypatch.setattr(R, "unrotate_f64", lambda y, sig: R.rotate_f64(y, sig))
    assert not mse_pin_holds()


def test_missing_codebook_scale_is_caught(monkeypatch):
    real = cb.lloyd_max_gauss
    monkeypatch.setattr(cb, "codebook", lambda d, bits, dist="gauss": (
        (real(1 << bits)).astype(np.float32), (0.5 * (real(1 << bits)[:-1] + real(1 << bits)[1:])).astype(np.float32),
        real(1 << bits), 0.5 * (real(1 << bits)[:-1] + real(1 << bits)[1:])))
    assert not mse_pin_holds()


def test_dropped_qjl_term_is_caught(monkeypatch):
    real = Q.rotated_estimate

    def mutant(qz, enc):
        if not qz.prod:
            return real(qz, enc)
        idx = Q.unpack_bits(enc["codes"], qz.d, qz.bm)
        return qz.centroids.astype(np.float64)[idx]  # the residual correction dropped

    monkeypatch.setattr(Q, "rotated_estimate", mutant)
    assert not prod_unbiased_pin_holds()


def test_flipped_qjl_sign_is_caught(monkeypatch):
    real = Q.rotated_estimate

    def mutant(qz, enc):
        flipped = dict(enc)
        flipped["qjl"] = np.bitwise_not(enc["qjl"])
        return real(qz, flipped)

    monkeypatch.setattr(Q, "rotated_estimate", mutant)
    assert not prod_unbiased_pin_holds()


def test_transposed_qjl_matrix_is_caught(monkeypatch):
    real = Q.rotated_estimate

    def mutant(qz, enc):
        qz2 = Q.Quantizer(qz.d, qz.bits, qz.variant, qz.seed_rot, qz.seed_qjl)
        qz2.S = np.ascontiguousarray(qz.S.T)  # S^T used where S belongs
        return real(qz2, enc)

    monkeypatch.setattr(Q, "rotated_estimate", mutant)
    assert not prod_unbiased_pin_holds()


def test_missing_softmax_scale_is_caught(monkeypatch):
    real = OA.dense_attention
    monkeypatch.setattr(OA, "dense_attention", lambda q, K, V, scale=None: real(q, K, V, scale=1.0))
    assert not attention_definition_pin_holds()
