"""GPU top-k vector search (tq_search_topk) against the oracle's search.

The device scores with the decode kernel's fp16 hi/lo tensor-core estimator,
the oracle in float64 on its own encoding of the same database (the codes
agree bit for bit: see the encode tests).  Where two records' estimates are
closer than the scoring error the order between them is not unique, so the
test compares what is: every returned index is a valid, distinct record; its
returned estimate equals the oracle's within the scores' tolerance; it ranks
within that tolerance of the oracle's k-th best; and the returned estimates
are ordered."""

import numpy as np
import pytest
import torch

from kv_cache_vector_13_b200 import api
from oracle import quantizer as OQ
from oracle import search as OS

from helpers import host, oracle_twin

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check(top_v, top_i, est, k):
    n_q, N = est.shape
    kk = min(k, N)
    for i in range(n_q):
        idx = top_i[i, :kk]
        assert np.all((idx >= 0) & (idx < N)) and len(set(idx.tolist())) == kk
        tol = 2e-3 * np.abs(est[i]).max()
        np.testing.assert_allclose(top_v[i, :kk], est[i, idx], rtol=0, atol=tol)
        kth = np.sort(est[i])[::-1][kk - 1]
        assert np.all(est[i, idx] >= kth - 2 * tol)
        assert np.all(np.diff(top_v[i, :kk]) <= 0)
        if kk < k:
            assert np.all(top_i[i, kk:] == -1) and np.all(np.isneginf(top_v[i, kk:]))


@pytest.mark.parametrize("bits,variant,rotation", [(4, "mse", "hadamard"), (3, "prod", "hadamard"),
                                                   (2, "mse", "hadamard"), (3, "mse", "dense")])
@pytest.mark.parametrize("n_q", [3, 13])
def test_search_topk_matches_oracle(bits, variant, rotation, n_q):
    N, d, k = 5000 + 17, 128, 10
    g = torch.Generator().manual_seed(bits * 100 + n_q)
    X = torch.randn((N, d), generator=g)
    Q = torch.randn((n_q, d), generator=g).to(torch.bfloat16)
    qz = api.Quantizer(d, bits, variant, seed_rot=5, seed_qjl=6, device=DEV, rotation=rotation)
    db = api.encode(qz, X.to(DEV))
    tv, ti = api.search_topk(qz, Q.to(DEV), db, k)
    oq = oracle_twin(qz)
    enc = OQ.encode(oq, host(X), aux=False)
    est = OS.scores(oq, host(Q), enc)
    check(host(tv), host(ti), est, k)


@pytest.mark.parametrize("k", [1, 32])
def test_search_k_extremes_and_short_database(k):
    d = 128
    g = torch.Generator().manual_seed(k)
    for N in (20, 3000):
        X = torch.randn((N, d), generator=g)
        Q = torch.randn((5, d), generator=g)
        qz = api.Quantizer(d, 4, "mse", seed_rot=8, device=DEV)
        tv, ti = api.search_topk(qz, Q.to(DEV), api.encode(qz, X.to(DEV)), k)
        oq = oracle_twin(qz)
        est = OS.scores(oq, host(Q), OQ.encode(oq, host(X), aux=False))
        check(host(tv), host(ti), est, k)


def test_search_finds_the_nearest_neighbour_of_perturbed_members():
    # unit database, queries are slightly perturbed members: the top-1 is
    # the member (as the oracle also finds, see its pins)
    N, d = 100000, 128
    g = torch.Generator().manual_seed(1)
    X = torch.randn((N, d), generator=g)
    X /= X.norm(dim=1, keepdim=True)
    members = torch.tensor([5, 12345, 99999, 50000])
    Q = X[members] + 0.01 * torch.randn((4, d), generator=g)
    qz = api.Quantizer(d, 4, "mse", seed_rot=9, device=DEV)
    tv, ti = api.search_topk(qz, Q.to(DEV), api.encode(qz, X.to(DEV)), 5)
    assert host(ti)[:, 0].tolist() == members.tolist()
