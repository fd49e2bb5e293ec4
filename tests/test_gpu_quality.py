"""Quality of the GPU encode + dequant on the encode sweep (config 4), against
what the pages print (CPU oracle pins fix the same quantities for the oracle):

- TurboQuant_mse distortion on unit vectors lies between 1/4^b and
  2.72/4^b ("The Distortion Guarantee", Theorem 1 and the lower bound) and
  near the printed 0.36 / 0.117 / 0.030 / 0.009;
- the TurboQuant_prod inner-product estimate is unbiased ("I Spent 31 Hours
  On The Math Behind Turboquant", property 1);
- the mse estimate shrinks towards zero by a constant factor, so its bias
  grows with the true inner product, 0.01 -> 0.17 ("TurboQuant của Google",
  Fig. 2 discussion); at b = 1 the factor is 2/pi ("内存厂商的噩梦来了",
  section 3).
Random inputs come from seeded torch generators on the GPU; the metrics are
float64 torch reductions of the kernels' outputs."""

import math

import pytest
import torch

from kv_cache_vector_13_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"
PRINTED = {1: 0.36, 2: 0.117, 3: 0.030, 4: 0.009}


def unit_rows(n, d, g):
    x = torch.randn((n, d), generator=g, device=DEV, dtype=torch.float64)
    return x / x.norm(dim=1, keepdim=True)


def pairs(n, d, rho, g):
    """Unit rows x and q with <x, q> = rho exactly."""
    x = unit_rows(n, d, g)
    z = torch.randn((n, d), generator=g, device=DEV, dtype=torch.float64)
    z -= (z * x).sum(dim=1, keepdim=True) * x
    z /= z.norm(dim=1, keepdim=True)
    return x, rho * x + math.sqrt(1.0 - rho * rho) * z


def recon(qz, x):
    cache = api.encode(qz, x.float())
    return api.dequant(qz, cache)[0, 0].double()


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_mse_distortion_between_the_bounds(d, b):
    g = torch.Generator(device=DEV).manual_seed(1000 + 10 * d + b)
    x = unit_rows(1 << 14, d, g)
    qz = api.Quantizer(d, b, "mse", seed_rot=d + b, device=DEV)
    err = ((x - recon(qz, x)) ** 2).sum(dim=1)
    m, se = err.mean().item(), (err.std() / math.sqrt(err.numel())).item()
    assert 1.0 / 4 ** b < m - 4 * se and m + 4 * se < 2.72 / 4 ** b
    if d == 128:  # the printed values (b = 3 prints 0.030; the sphere integral is 0.034)
        assert abs(m - PRINTED[b]) <= 0.15 * PRINTED[b] + 4 * se


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_prod_inner_product_unbiased(d, b):
    g = torch.Generator(device=DEV).manual_seed(2000 + 10 * d + b)
    errs = []
    for seed in range(4):
        x, q = pairs(4096, d, 0.3, g)
        qz = api.Quantizer(d, b, "prod", seed_rot=seed, seed_qjl=100 + seed, device=DEV)
        errs.append((q * recon(qz, x)).sum(dim=1) - (q * x).sum(dim=1))
    e = torch.cat(errs)
    assert abs(e.mean().item()) < 4 * e.std().item() / math.sqrt(e.numel())


@pytest.mark.parametrize("b", [1, 2])
def test_mse_bias_grows_with_the_inner_product(b):
    # bias(rho) = -(1 - s) rho for one shrink factor s: linear in rho, and
    # s = 2/pi at b = 1; the prod estimate stays unbiased at every rho
    d = 128
    g = torch.Generator(device=DEV).manual_seed(3000 + b)
    qm = api.Quantizer(d, b, "mse", seed_rot=5, device=DEV)
    qp = api.Quantizer(d, b, "prod", seed_rot=6, seed_qjl=7, device=DEV)
    rhos = [0.01, 0.05, 0.1, 0.17]
    bias, se = [], []
    for rho in rhos:
        x, q = pairs(1 << 15, d, rho, g)
        e = (q * recon(qm, x)).sum(dim=1) - rho
        bias.append(e.mean().item())
        se.append(e.std().item() / math.sqrt(e.numel()))
        ep = (q * recon(qp, x)).sum(dim=1) - rho
        assert abs(ep.mean().item()) < 4 * ep.std().item() / math.sqrt(ep.numel())
    # least-squares shrink through the origin, then every point on the line
    s = 1.0 - sum(-bi * r for bi, r in zip(bias, rhos)) / sum(r * r for r in rhos)
    for bi, r, si in zip(bias, rhos, se):
        assert abs(bi + (1.0 - s) * r) < 4 * si + 1e-4
    assert abs(bias[-1]) > abs(bias[0])
    if b == 1:
        assert abs(s - 2.0 / math.pi) < 0.02
