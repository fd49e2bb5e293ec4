"""GPU parity of the dense (Haar) rotation option against the oracle.

The device computes u = fl(Pi x) * fl(1/n) with fp32 FMAs; the oracle takes
the exact product in float64.  So:
- norms are bit-exact (the same canonical fp32 fold-halves sum);
- a code may differ from the oracle's only for a coordinate whose exact u
  lies within the device's rounding band of a threshold,
  band = (6 d + 16) 2^-24 sum_k |Pi_jk x_k| / n + 2^-22 |u|
  (the tensor-core path: x and Pi each carried to 22 bits by fp16 halves,
  three products, 3d fp32 additions that may truncate; the CUDA-core path's
  fp32 dot product is well inside it); every such difference is checked
  against it and the count is reported;
- prod: the residual is the one the device's own indices give (an index
  that flipped inside the band moves its coordinate of r by a centroid
  step); ||r|| within 1e-5 relative of that residual's norm, and a QJL sign
  may differ only where |(S r)_k| is within the fp32 dot-product band plus
  what the residual's band and flipped indices can move it.
Decode attention with dense keys and values (d = 128) is compared with the
fp32 oracle at the 2e-3 tolerance of the other decode tests.
"""

import numpy as np
import pytest
import torch

from kv_cache_vector_13_b200 import api
from oracle import quantizer as OQ

from helpers import flat_host, host, oracle_attention, oracle_cache_slices, oracle_twin, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def u_band(oq, x):
    x = x.astype(np.float64)
    n = np.sqrt(np.sum(x * x, axis=1))
    P = oq.Pi.astype(np.float64)
    absdot = np.abs(x) @ np.abs(P).T
    u = (x @ P.T) / np.where(n > 0, n, 1.0)[:, None]
    band = (6 * oq.d + 16) * 2.0 ** -24 * absdot / np.where(n > 0, n, 1.0)[:, None] + 2.0 ** -22 * np.abs(u)
    return band


def check_dense_records(qz, oq, x, got):
    enc = OQ.encode(oq, x)
    np.testing.assert_array_equal(got["norms"].reshape(-1).view(np.uint32), enc["norms"].view(np.uint32))
    n, d = x.shape
    band = u_band(oq, x)
    nd = 0
    if qz.bm > 0:
        gi = OQ.unpack_bits(got["codes"].reshape(enc["codes"].shape), d, qz.bm)
        oi = OQ.unpack_bits(enc["codes"], d, qz.bm)
        diff = gi != oi
        nd = int(diff.sum())
        if nd:
            t = oq.thresholds.astype(np.float64)
            gap = np.abs(enc["u"][:, :, None] - t[None, None, :]).min(axis=2)
            assert np.all(gap[diff] <= band[diff]), "a code differs outside the rounding band"
    nq = 0
    if qz.prod:
        # the residual the device formed: the exact u with the device's own
        # indices (they differ from the oracle's only inside the band above,
        # and a flipped index moves that coordinate of r by a centroid step)
        gidx = (OQ.unpack_bits(got["codes"].reshape(enc["codes"].shape), d, qz.bm) if qz.bm else
                np.zeros((n, d), np.int64))
        c64 = oq.centroids.astype(np.float64)
        r = enc["u"] - (c64[OQ.unpack_bits(enc["codes"], d, oq.bm)] if oq.bm else 0.0)
        r_dev = enc["u"] - (c64[gidx] if oq.bm else 0.0)
        g = got["rnorms"].reshape(-1).astype(np.float64)
        want = np.sqrt(np.sum(r_dev ** 2, axis=1))
        assert np.all(np.abs(g - want) <= 1e-5 * np.maximum(want, 1e-30) + 4 * d * 2.0 ** -24 * np.sqrt(
            np.sum(band ** 2, axis=1)))
        gq = OQ.unpack_bits(got["qjl"].reshape(enc["qjl"].shape), d, 1)
        oqb = OQ.unpack_bits(enc["qjl"], d, 1)
        qd = gq != oqb
        nq = int(qd.sum())
        if nq:
            S = np.abs(oq.S.astype(np.float64))
            zb = ((d + 2) * 2.0 ** -24 * (np.abs(r) @ S.T)
                  + (band + 2.0 ** -23 * np.abs(r) + np.abs(r_dev - r)) @ S.T)
            assert np.all(np.abs(enc["z"])[qd] <= zb[qd]), "a QJL sign differs outside its band"
    return nd, nq


@pytest.mark.parametrize("d", [64, 128, 200, 256])
@pytest.mark.parametrize("bits,variant", [(2, "mse"), (4, "mse"), (3, "prod")])
def test_dense_encode_matches_oracle(d, bits, variant):
    n = 3000
    g = torch.Generator().manual_seed(d * 10 + bits)
    x = torch.randn((n, d), generator=g) * torch.exp(torch.randn((n, 1), generator=g))
    x[::101] = 0.0
    qz = api.Quantizer(d, bits, variant, seed_rot=40 + d, seed_qjl=41, device=DEV, rotation="dense")
    cache = api.encode(qz, x.to(DEV))
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    nd, nq = check_dense_records(qz, oq, host(x), flat_host(cache))
    assert nd <= max(4, 2e-5 * n * d) and nq <= max(4, 2e-5 * n * d), (nd, nq)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_dense_encode_half_inputs_strided(dtype):
    B, N, H, d = 2, 500, 3, 128
    g = torch.Generator().manual_seed(3)
    buf = (torch.randn((B, N, H, d), generator=g) * 3).to(dtype)
    x = buf.permute(0, 2, 1, 3)
    qz = api.Quantizer(d, 4, "mse", seed_rot=44, device=DEV, rotation="dense")
    cache = api.encode(qz, x.to(DEV))
    torch.cuda.synchronize()
    check_dense_records(qz, oracle_twin(qz), host(x).reshape(-1, d), flat_host(cache))


@pytest.mark.parametrize("d,bits,variant", [(64, 3, "mse"), (200, 2, "prod"), (256, 4, "mse")])
def test_dense_dequant_matches_oracle(d, bits, variant):
    n = 700
    x = torch.randn((n, d), generator=torch.Generator().manual_seed(d))
    qz = api.Quantizer(d, bits, variant, seed_rot=50, seed_qjl=51, device=DEV, rotation="dense")
    cache = api.encode(qz, x.to(DEV))
    xh = host(api.dequant(qz, cache)).reshape(n, d)
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x))
    ref = OQ.dequant(oq, enc)
    # rows whose records equal the oracle's (all but the few with a code or
    # sign inside the rounding band) reconstruct to the same vector
    got = flat_host(cache)
    same = np.ones(n, bool)
    for k in ("codes", "qjl"):
        if k in enc:
            same &= np.all(got[k].reshape(enc[k].shape) == enc[k], axis=1)
    assert same.mean() > 0.99
    nrm = enc["norms"].astype(np.float64)[:, None]
    assert np.all((np.abs(xh - ref) <= 4 * d * 2.0 ** -24 * nrm + 1e-30)[same])


@pytest.mark.parametrize("kspec,vspec", [((4, "mse"), (4, "mse")), ((3, "prod"), (3, "mse"))])
def test_dense_decode_matches_oracle(kspec, vspec):
    B, Hq, Hkv, N, d = 2, 8, 2, 1500, 128
    g = torch.Generator(device=DEV).manual_seed(61)
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
    kq = api.Quantizer(d, kspec[0], kspec[1], seed_rot=62, seed_qjl=63, device=DEV, rotation="dense")
    vq = api.Quantizer(d, vspec[0], vspec[1], seed_rot=64, device=DEV, rotation="dense")
    kc, vc = api.encode(kq, K), api.encode(vq, V)
    out = host(api.decode_attention(kq, vq, q, kc, vc))
    okq, ovq = oracle_twin(kq), oracle_twin(vq)
    okc, _ = oracle_cache_slices(okq, host(K))
    ovc, _ = oracle_cache_slices(ovq, host(V))
    ref = oracle_attention(okq, ovq, host(q), okc, ovc)
    assert rel_err(out, ref).max() <= 2e-3
