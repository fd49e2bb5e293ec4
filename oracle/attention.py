"""Decode attention on the packed TurboQuant cache (oracle side; test
infrastructure).

Attention for one new query: softmax(q K^T / sqrt(d)) V over every cached
token ("I Spent 31 Hours On The Math Behind Turboquant", section "KV Cache:
The problem"; HN thread on TurboQuant, the single-head decoder walk-through).
Keys are scored with the asymmetric estimator: a full-precision query against
compressed keys ("内存厂商的噩梦来了", sections 4.2 and the pseudocode
function asymmetric_attention_score), i.e. for key j

    est_j = n_j * ( <q', c[idx_j]> + gamma_j * sqrt(pi/2)/d * <S q', sign_j> )

with q' = Pi q the query in the rotated basis (the prod term only for
TurboQuant_prod keys; Pi is the randomized Hadamard map or, for the dense
option, the stored Haar matrix).  Reading: the pseudocode's correction has no scale and
no ||r||; the scale sqrt(pi/2)/d * ||r|| that makes the QJL estimate unbiased
for m = d projections is used instead ("TurboQuant của Google", section "Vấn
đề của inner product", the unbiased QJL estimator).

Values are summed in the rotated basis, o' = sum_j p_j n_j c_V[idx_j], and
rotated back once, o = Pi_V^T o'.  No causal mask: the decode query sees the
whole cache.
"""

import math

import numpy as np

from . import quantizer as _qz
from . import rotation as _rot

LOG2E = 1.4426950408889634


_CHUNK = 1 << 16


def _scores_one(qz, q, cache, dtype=np.float64):
    """Estimator <q, k_j> for every token of one (batch, kv head) slice.

    ``cache``: dict(codes [N, nb], norms [N], qjl, rnorms) for that slice.
    Tokens are unpacked in chunks only to bound memory.
    """
    f = dtype
    d = qz.d
    N = cache["norms"].shape[0]
    sig = qz.signs.astype(f)
    if qz.dense:
        qp = qz.Pi.astype(f) @ np.asarray(q, f)
    elif f == np.float64:
        qp = _rot.rotate_f64(q, qz.signs)
    else:
        qp = _rot.fwht_f32((np.asarray(q, np.float32) * sig)[None, :])[0] / np.float32(math.sqrt(d))
    qs = qz.S.astype(f) @ qp.astype(f) if qz.prod else None
    out = np.empty(N, f)
    for lo in range(0, N, _CHUNK):
        hi = min(N, lo + _CHUNK)
        n = cache["norms"][lo:hi].astype(f)
        if qz.bm > 0:
            idx = _qz.unpack_bits(cache["codes"][lo:hi], d, qz.bm)
            main = qz.centroids.astype(f)[idx] @ qp.astype(f)
        else:
            main = np.zeros(hi - lo, f)
        if qz.prod:
            sg = (2 * _qz.unpack_bits(cache["qjl"][lo:hi], d, 1) - 1).astype(f)
            gam = cache["rnorms"][lo:hi].astype(f)
            main = main + gam * f(_qz.SQRT_HALF_PI / d) * (sg @ qs)
        out[lo:hi] = n * main
    return out


def _values_one(vq, p, cache, dtype=np.float64):
    """Pi_V^T sum_j p_j v_hat_rot_j n_j for one slice (p already normalised)."""
    f = dtype
    d = vq.d
    N = cache["norms"].shape[0]
    op = np.zeros(d, f)
    for lo in range(0, N, _CHUNK):
        hi = min(N, lo + _CHUNK)
        w = (p[lo:hi] * cache["norms"][lo:hi].astype(f)).astype(f)
        if vq.bm > 0:
            idx = _qz.unpack_bits(cache["codes"][lo:hi], d, vq.bm)
            op = op + w @ vq.centroids.astype(f)[idx]
        if vq.prod:
            sg = (2 * _qz.unpack_bits(cache["qjl"][lo:hi], d, 1) - 1).astype(f)
            gam = cache["rnorms"][lo:hi].astype(f)
            op = op + ((w * gam) @ sg) @ vq.S.astype(f) * f(_qz.SQRT_HALF_PI / d)
    if vq.dense:
        return op.astype(f) @ vq.Pi.astype(f)          # Pi^T o'
    if f == np.float64:
        return _rot.unrotate_f64(op, vq.signs)
    sig = vq.signs.astype(np.float32)
    return sig * _rot.fwht_f32(op.astype(np.float32)[None, :])[0] / np.float32(math.sqrt(d))


def slice_cache(enc: dict, b: int, h: int) -> dict:
    """Select one (batch, kv head) slice of a cache dict whose arrays are
    shaped [B, Hkv, N, ...]."""
    return {k: v[b, h] for k, v in enc.items() if v is not None}


def decode_attention(kq, vq, q, kcache, vcache, scale=None, dtype=np.float64,
                     heads=None, return_scores=False):
    """Decode attention for queries q [B, Hq, d] over packed caches whose
    arrays are shaped [B, Hkv, N, ...].  GQA: query head hq reads kv head
    hq // (Hq // Hkv).  ``heads``: optional list of (b, hq) to compute
    (others are left zero).  Returns out [B, Hq, d] (and the pre-scale
    estimator scores [B, Hq, N] when ``return_scores``).
    """
    f = dtype
    B, Hq, d = q.shape
    Hkv = kcache["norms"].shape[1]
    N = kcache["norms"].shape[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((B, Hq, d), f)
    scores = np.zeros((B, Hq, N), f) if return_scores else None
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for (b, hq) in todo:
        h = hq // g
        kc = slice_cache(kcache, b, h)
        vc = slice_cache(vcache, b, h)
        s = _scores_one(kq, np.asarray(q[b, hq], f), kc, dtype=f)
        if return_scores:
            scores[b, hq] = s
        if N == 0:
            continue
        logits = s * f(scale)
        m = logits.max()
        e = np.exp(logits - m)
        p = e / e.sum()
        out[b, hq] = _values_one(vq, p, vc, dtype=f)
    if return_scores:
        return out, scores
    return out


def dense_attention(q, K, V, scale=None):
    """Plain float64 softmax(q K^T * scale) V for one query [d] against
    K, V [N, d] (used to pin the packed-cache path against its definition)."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[0])
    logits = K @ q * scale
    e = np.exp(logits - logits.max())
    return (e / e.sum()) @ V
