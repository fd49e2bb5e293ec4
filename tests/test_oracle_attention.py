"""Pins for the oracle's decode attention on the packed cache (CPU)."""

import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import quantizer as Q


def brute_attention(q, K, V, scale):
    """softmax(q . k_j * scale) weighted sum of v_j, in plain Python loops."""
    logits = [scale * sum(qi * ki for qi, ki in zip(q, k)) for k in K]
    m = max(logits)
    e = [math.exp(l - m) for l in logits]
    tot = sum(e)
    return [sum(e[j] / tot * V[j][i] for j in range(len(K))) for i in range(len(q))]


def test_dense_attention_is_the_definition():
    rng = np.random.default_rng(0)
    q, K, V = rng.standard_normal(8), rng.standard_normal((5, 8)), rng.standard_normal((5, 8))
    want = brute_attention(q.tolist(), K.tolist(), V.tolist(), 1 / math.sqrt(8))
    np.testing.assert_allclose(A.dense_attention(q, K, V), want, rtol=1e-12)


def make_cache(qz, X):
    """Encode X [B, Hkv, N, d] into cache arrays shaped [B, Hkv, N, ...]."""
    B, H, N, d = X.shape
    enc = Q.encode(qz, X.reshape(-1, d))
    out = {}
    for k in ("codes", "norms", "qjl", "rnorms"):
        if k in enc:
            v = enc[k]
            out[k] = v.reshape((B, H, N) + v.shape[1:])
    return out, Q.dequant(qz, enc).reshape(B, H, N, d)


@pytest.mark.parametrize("kvar,kb,vvar,vb,d", [("mse", 4, "mse", 4, 128), ("prod", 3, "mse", 3, 128),
                                               ("prod", 4, "mse", 4, 128), ("mse", 3, "mse", 2, 128),
                                               ("prod", 3, "prod", 3, 64), ("mse", 2, "prod", 4, 256),
                                               ("prod", 1, "prod", 1, 64)])
def test_packed_attention_equals_attention_on_dequantized_cache(kvar, kb, vvar, vb, d):
    # prod values: the values are summed in the rotated basis and S^T is
    # applied once to the weighted sign sums; the result must equal
    # attention over the dequantized values x_hat = n Pi^T (c + gamma
    # sqrt(pi/2)/d S^T sign)
    rng = np.random.default_rng(kb * 10 + vb + d)
    B, Hq, Hkv, N = 2, 8, 2, 300
    kq = Q.Quantizer(d, kb, kvar, seed_rot=1, seed_qjl=2)
    vq = Q.Quantizer(d, vb, vvar, seed_rot=3, seed_qjl=4)
    K = (rng.standard_normal((B, Hkv, N, d)) * rng.lognormal(0, 0.5, (1, Hkv, 1, d))).astype(np.float32)
    V = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    q = rng.standard_normal((B, Hq, d))
    kc, Kh = make_cache(kq, K)
    vc, Vh = make_cache(vq, V)
    out, scores = A.decode_attention(kq, vq, q, kc, vc, return_scores=True)
    g = Hq // Hkv
    for b in range(B):
        for hq in range(Hq):
            h = hq // g
            np.testing.assert_allclose(scores[b, hq], Kh[b, h] @ q[b, hq], rtol=1e-9, atol=1e-9)
            np.testing.assert_allclose(out[b, hq], A.dense_attention(q[b, hq], Kh[b, h], Vh[b, h]),
                                       rtol=1e-9, atol=1e-9)


def test_fp32_oracle_tracks_float64():
    rng = np.random.default_rng(3)
    B, Hq, Hkv, N, d = 1, 4, 1, 2000, 128
    kq = Q.Quantizer(d, 3, "prod", seed_rot=5, seed_qjl=6)
    vq = Q.Quantizer(d, 3, "mse", seed_rot=7)
    K = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    q = rng.standard_normal((B, Hq, d))
    kc, _ = make_cache(kq, K)
    vc, _ = make_cache(vq, V)
    o64 = A.decode_attention(kq, vq, q, kc, vc)
    o32 = A.decode_attention(kq, vq, q.astype(np.float32), kc, vc, dtype=np.float32)
    err = np.abs(o32 - o64).max(axis=2) / np.abs(o64).max(axis=2)
    assert err.max() < 1e-5


def test_more_bits_approach_exact_attention():
    rng = np.random.default_rng(4)
    N, d = 512, 64
    K = rng.standard_normal((1, 1, N, d)).astype(np.float32) * 2
    V = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    q = rng.standard_normal((1, 1, d))
    exact = A.dense_attention(q[0, 0], K[0, 0], V[0, 0])
    errs = []
    for b in (1, 2, 3, 4):
        kq, vq = Q.Quantizer(d, b, seed_rot=1), Q.Quantizer(d, b, seed_rot=2)
        kc, _ = make_cache(kq, K)
        vc, _ = make_cache(vq, V)
        errs.append(np.abs(A.decode_attention(kq, vq, q, kc, vc)[0, 0] - exact).max())
    assert errs[3] < errs[1] < errs[0]
