"""GPU parity of tq_encode / tq_dequant against the oracle (bit-exact codes)."""

import math

import numpy as np
import pytest
import torch

from kv_cache_vector_13_b200 import api, inputs
from oracle import quantizer as OQ

from helpers import compare_records, flat_host, host, oracle_twin

pytestmark = pytest.mark.gpu
DEV = "cuda"


def sample_vectors(n, d, seed, dtype):
    """Gaussian rows with per-row scales over several decades, exact zeros,
    and rows scaled by 1e12 and 1e-12 (all squares stay finite and normal)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((n, d), generator=g)
    x *= torch.exp(torch.randn((n, 1), generator=g) * 2.0).clamp(1e-3, 1e3)
    x[::97] = 0.0
    x[5::131] *= 1e12
    x[7::131] *= 1e-12
    return x.to(dtype)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits,variant", [(1, "mse"), (2, "mse"), (3, "mse"), (4, "mse"),
                                          (1, "prod"), (2, "prod"), (3, "prod"), (4, "prod")])
def test_encode_bit_exact_fp32(d, bits, variant):
    n = 1000 + 37  # ragged: not a multiple of any block
    x = sample_vectors(n, d, 11 * d + bits, torch.float32)
    qz = api.Quantizer(d, bits, variant, seed_rot=3, seed_qjl=4, device=DEV)
    cache = api.encode(qz, x.to(DEV))
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x))
    nd = compare_records(qz, oq, enc, flat_host(cache))
    assert nd <= 2


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits,variant", [(4, "mse"), (3, "mse"), (3, "prod"), (4, "prod")])
def test_encode_bit_exact_half_inputs_strided(dtype, bits, variant):
    # [B, N, H, d] buffer encoded through a [B, H, N, d] view into a [B, H, N] cache
    B, N, H, d = 2, 333, 3, 128
    g = torch.Generator().manual_seed(bits)
    buf = (torch.randn((B, N, H, d), generator=g) * 3).to(dtype)
    x = buf.permute(0, 2, 1, 3)
    qz = api.Quantizer(d, bits, variant, seed_rot=9, seed_qjl=10, device=DEV)
    cache = api.encode(qz, x.to(DEV))
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x).reshape(-1, d))
    compare_records(qz, oq, enc, flat_host(cache))


@pytest.mark.parametrize("bits", [3, 4])
def test_encode_bit_exact_bf16_large_batch_strided(bits):
    # more than 18944 vectors take the 64-coordinates-per-lane layout: the
    # one that encodes the decode workloads' bf16 K and V from a
    # [B, N, H, d] projection buffer through a [B, H, N, d] view
    B, N, H, d = 2, (1 << 15) + 17, 2, 128
    g = torch.Generator(device=DEV).manual_seed(60 + bits)
    buf = (torch.randn((B, N, H, d), generator=g, device=DEV) * 2).to(torch.bfloat16)
    buf[:, ::1001] = 0
    x = buf.permute(0, 2, 1, 3)
    qz = api.Quantizer(d, bits, "mse", seed_rot=61, device=DEV)
    cache = api.encode(qz, x)
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x).reshape(-1, d), chunk=1 << 15, aux=False)
    compare_records(qz, oq, enc, flat_host(cache))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 3])
def test_encode_bit_exact_fp32_large_batch(d, bits):
    # the large-batch layout at every d, for the b_m values the other large
    # tests leave out (1: the sign bit alone; 3: fields that straddle words)
    n = (1 << 16) + 37
    x = sample_vectors(n, d, 7 * d + bits, torch.float32)
    qz = api.Quantizer(d, bits, "mse", seed_rot=70 + bits, device=DEV)
    cache = api.encode(qz, x.to(DEV))
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x), chunk=1 << 15, aux=False)
    compare_records(qz, oq, enc, flat_host(cache))


def test_encode_into_strided_cache_and_tail_append():
    # cache layout [B, H, Ncap] written one token at a time (decode-step append)
    B, H, Ncap, d = 2, 4, 40, 128
    qz = api.Quantizer(d, 4, "mse", seed_rot=1, device=DEV)
    cache = api.empty_cache(qz, B, H, Ncap, DEV)
    cache.norms.fill_(-7.0)
    X = torch.randn((B, H, Ncap, d), device=DEV)
    for n in range(Ncap):
        sub = api.PackedCache(cache.codes[:, :, n:n + 1], cache.norms[:, :, n:n + 1])
        api.encode(qz, X[:, :, n:n + 1], out=sub)
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(X).reshape(-1, d))
    compare_records(qz, oq, enc, flat_host(cache))


def test_encode_config4_full_size_d128_b4():
    # 2^20 unit vectors, the encode roofline workload, every record checked
    d, n = 128, 1 << 20
    x = inputs.unit_vectors(n, d, seed=0, device=DEV)
    qz = api.Quantizer(d, 4, "mse", seed_rot=0, device=DEV)
    cache = api.encode(qz, x)
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x), chunk=1 << 15)
    compare_records(qz, oq, enc, flat_host(cache))


@pytest.mark.parametrize("d,bits,variant", [(64, 3, "prod"), (128, 3, "prod"), (256, 2, "prod"), (128, 2, "mse")])
def test_encode_config4_sampled_sizes(d, bits, variant):
    n = 1 << 16
    x = inputs.unit_vectors(n, d, seed=1, device=DEV)
    qz = api.Quantizer(d, bits, variant, seed_rot=0, seed_qjl=1, device=DEV)
    cache = api.encode(qz, x)
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x))
    nd = compare_records(qz, oq, enc, flat_host(cache))
    if variant == "prod":
        assert nd <= max(2, 1e-6 * n * d)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits,variant", [(3, "mse"), (4, "mse"), (1, "prod"), (3, "prod")])
def test_dequant_matches_oracle(d, bits, variant):
    n = 777
    x = sample_vectors(n, d, 5, torch.float32)
    qz = api.Quantizer(d, bits, variant, seed_rot=21, seed_qjl=22, device=DEV)
    cache = api.encode(qz, x.to(DEV))
    xh = host(api.dequant(qz, cache))
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x))
    ref = OQ.dequant(oq, enc)
    nrm = enc["norms"].astype(np.float64)[:, None]
    # fp32 butterflies and projections against float64: a few ulps of ||x||,
    # plus one QJL term for a sign that may differ at the rounding boundary
    tol = 2e-6 * math.log2(d) * nrm + (1.0 if variant == "prod" else 0.0) * 3 * math.sqrt(math.pi / 2) / d * nrm
    assert np.all(np.abs(xh.reshape(n, d) - ref) <= tol + 1e-30)


def test_zero_and_empty_inputs():
    qz = api.Quantizer(128, 3, "prod", device=DEV)
    x = torch.zeros((5, 128), device=DEV)
    cache = api.encode(qz, x)
    # n = 0 gives u = 0, the middle index, a residual of -c[K/2-1] and x_hat = 0
    assert torch.all(cache.norms == 0)
    assert torch.all(api.dequant(qz, cache) == 0)
    empty = api.encode(qz, torch.zeros((0, 128), device=DEV))
    assert empty.norms.numel() == 0
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("bits", [1, 2, 4])
def test_encode_prod_large_batch_projection(dtype, bits):
    # d = 128 prod batches of more than a wave take the tensor-core QJL
    # projection; a ragged last tile, a zero row (zero residual for b = 1)
    # and a tiny-norm row ride along.  Codes, norms and residual norms stay
    # bit-exact; QJL signs may differ only inside the fp32 band.
    d, n = 128, 3 * (1 << 13) + 37
    x = inputs.unit_vectors(n, d, seed=bits, device=DEV)
    x[5] = 0.0
    x[6] *= 1e-30
    x = x.to(dtype)
    qz = api.Quantizer(d, bits, "prod", seed_rot=50 + bits, seed_qjl=60 + bits, device=DEV)
    cache = api.encode(qz, x)
    torch.cuda.synchronize()
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(x))
    nd = compare_records(qz, oq, enc, flat_host(cache))
    assert nd <= max(2, 1e-6 * n * d)
