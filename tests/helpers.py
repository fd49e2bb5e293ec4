"""Shared helpers for the GPU parity tests: oracle twins of device
quantizers, and record comparison with the QJL boundary allowance."""

import numpy as np
import torch

from oracle import attention as OA
from oracle import quantizer as OQ


def oracle_twin(qz) -> OQ.Quantizer:
    """The oracle's own quantizer with the same (d, bits, variant, seeds)."""
    return OQ.Quantizer(qz.d, qz.bits, qz.variant, seed_rot=qz.seed_rot, seed_qjl=qz.seed_qjl, dist=qz.dist,
                        rotation=qz.rotation)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16 or t.dtype == torch.float16:
        t = t.float()
    return t.detach().cpu().numpy()


def qjl_bound(oq: OQ.Quantizer, enc: dict) -> np.ndarray:
    """Forward-error bound of an fp32 summation of d products for every
    projection z_k = sum_i S_ki r_i: d * 2^-24 * sum_i |S_ki r_i| (rows =
    vectors).  A device sign may differ from the float64 sign only inside it."""
    idx = OQ.unpack_bits(enc["codes"], oq.d, oq.bm)
    r = enc["u"].astype(np.float64) - (oq.centroids.astype(np.float64)[idx] if oq.bm else 0.0)
    return oq.d * 2.0 ** -24 * (np.abs(r) @ np.abs(oq.S.astype(np.float64)).T)


def flat_host(cache, sl=None) -> dict:
    """Host copies of a device cache's arrays, flattened to [n, ...] in
    (b, h, n) order; ``sl`` = (b, h) keeps one slice."""
    out = {}
    for k in ("codes", "norms", "qjl", "rnorms"):
        t = getattr(cache, k)
        if t is None:
            continue
        a = host(t)
        if sl is not None:
            a = a[sl[0], sl[1]]
            out[k] = a
        else:
            out[k] = a.reshape((-1,) + a.shape[3:])
    return out


def compare_records(qz, oq, enc: dict, got: dict) -> int:
    """Codes, norms and residual norms bit-exact; QJL bits equal except inside
    the fp32 rounding band around zero.  ``got``: flat_host(...) of the device
    cache covering the same vectors as ``enc``.  Returns the number of QJL
    bits that differ (all of them inside the band)."""
    np.testing.assert_array_equal(got["norms"].reshape(-1).view(np.uint32), enc["norms"].view(np.uint32))
    if qz.bm > 0:
        codes = got["codes"].reshape(enc["codes"].shape)
        bad = np.nonzero(codes != enc["codes"])
        assert bad[0].size == 0, f"{bad[0].size} code bytes differ (first vectors {bad[0][:4]})"
    if not qz.prod:
        return 0
    np.testing.assert_array_equal(got["rnorms"].reshape(-1).view(np.uint32), enc["rnorms"].view(np.uint32))
    gq = OQ.unpack_bits(got["qjl"].reshape(enc["qjl"].shape), qz.d, 1)
    oqb = OQ.unpack_bits(enc["qjl"], qz.d, 1)
    diff = gq != oqb
    n = int(diff.sum())
    if n:
        band = qjl_bound(oq, enc)
        z = np.abs(enc["z"])
        assert np.all(z[diff] <= band[diff]), "a QJL sign differs outside the fp32 rounding band"
    return n


def rel_err(out: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """max |o - o_ref| / max |o_ref| over the last axis."""
    return np.abs(out - ref).max(axis=-1) / np.maximum(np.abs(ref).max(axis=-1), 1e-30)


def oracle_cache_slices(oq, X: np.ndarray, chunk=8192):
    """Oracle-encode X [B, H, N, d] into cache arrays shaped [B, H, N, ...]."""
    B, H, N, d = X.shape
    enc = OQ.encode(oq, X.reshape(-1, d), chunk=chunk, aux=False)
    out = {}
    for k in ("codes", "norms", "qjl", "rnorms"):
        if k in enc:
            v = enc[k]
            out[k] = v.reshape((B, H, N) + v.shape[1:])
    return out, enc


def oracle_attention(kq, vq, q, kc, vc, heads=None, scale=None):
    return OA.decode_attention(kq, vq, np.asarray(q, np.float32), kc, vc, scale=scale, dtype=np.float32,
                               heads=heads)


def compare_slice_records(qz, oq, X: np.ndarray, cache, b: int, h: int, chunk: int = 1 << 16) -> int:
    """Oracle-encode the rows X [N, d] of one (batch, kv head) slice chunk by
    chunk (with the auxiliary u and z the QJL band needs) and compare them
    with the device cache's records of slice (b, h).  Returns the number of
    QJL bits that differ (all inside the fp32 band)."""
    got_all = flat_host(cache, sl=(b, h))
    n = X.shape[0]
    nd = 0
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        enc = OQ.encode(oq, X[lo:hi], chunk=chunk)
        got = {k: v[lo:hi] for k, v in got_all.items()}
        nd += compare_records(qz, oq, enc, got)
    return nd
