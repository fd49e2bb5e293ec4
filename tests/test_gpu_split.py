"""GPU outlier-channel split against the oracle's: the page's example split
(32 outlier channels at 3 bits, 96 regular channels at 2 bits), outlier
channels chosen by the largest mean square over the first prefill block.
Each group's records follow the dense-rotation parity rule (norms bit-exact,
codes equal except inside the rounding band); split decode attention matches
the fp32 oracle within 2e-3."""

import numpy as np
import pytest
import torch

from kv_cache_vector_13_b200 import api
from oracle import split as SP

from helpers import flat_host, host, rel_err
from test_gpu_dense import check_dense_records

pytestmark = pytest.mark.gpu
DEV = "cuda"


def workload(B, Hkv, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    scale = torch.ones(d)
    scale[torch.randperm(d, generator=g)[:32]] = 8.0  # planted outlier channels
    K = torch.randn((B, Hkv, N, d), generator=g) * scale
    V = torch.randn((B, Hkv, N, d), generator=g) * scale
    return K, V


@pytest.mark.parametrize("kvariant", ["mse", "prod"])
def test_split_records_and_decode_match_oracle(kvariant):
    B, Hq, Hkv, N, d = 2, 8, 2, 900, 128
    K, V = workload(B, Hkv, N, d, seed=3)
    # channel selection on the first 64 tokens of batch 0, kv head 0
    ch = SP.select_outlier_channels(host(K[0, 0, :64]), 32)
    kq = api.SplitQuantizer(d, ch, 3, 2, kvariant, seed_rot=11, seed_qjl=12, device=DEV)
    vq = api.SplitQuantizer(d, ch, 3, 2, "mse", seed_rot=13, device=DEV)
    kc = api.encode_split(kq, K.to(DEV))
    vc = api.encode_split(vq, V.to(DEV))
    torch.cuda.synchronize()
    okq = SP.SplitQuantizer(d, ch, 3, 2, kvariant, seed_rot=11, seed_qjl=12)
    ovq = SP.SplitQuantizer(d, ch, 3, 2, "mse", seed_rot=13)
    # records of each group, bit for bit up to the rounding band
    Kh = host(K).reshape(-1, d)
    for gq, oq, idx, cache in ((kq.groups[0], okq.outlier, okq.channels, kc[0]),
                               (kq.groups[1], okq.regular, okq.rest, kc[1])):
        check_dense_records(gq, oq, np.ascontiguousarray(Kh[:, idx]), flat_host(cache))
    q = torch.randn((B, Hq, d), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    lens = torch.tensor([N, 517], dtype=torch.int32, device=DEV)
    op = api.DecodeAttentionSplit(kq, vq, B, Hq, Hkv, N, device=DEV)
    out = host(op(q.to(DEV), kc, vc, seq_lens=lens))
    g = Hq // Hkv
    qh = host(q)
    for b in range(B):
        L = int(lens[b])
        for h in range(Hkv):
            ke = SP.encode(okq, host(K[b, h, :L]), aux=False)
            ve = SP.encode(ovq, host(V[b, h, :L]), aux=False)
            for hq in range(h * g, (h + 1) * g):
                ref = SP.decode_attention(okq, ovq, qh[b, hq], ke, ve, dtype=np.float32)
                e = rel_err(out[b, hq], ref)
                assert e <= 2e-3, (b, hq, e)


def test_split_record_sizes_and_empty_cache():
    d = 128
    kq = api.SplitQuantizer(d, list(range(0, 128, 4)), 3, 2, "mse", device=DEV)
    assert kq.groups[0].code_bytes == 12 and kq.groups[1].code_bytes == 24
    caches = api.encode_split(kq, torch.zeros((0, d), device=DEV))
    assert caches[0].norms.numel() == 0


def test_split_decode_twelve_query_heads_per_kv_head():
    # a GQA group of 12 (two head groups of a block) and prod value groups
    B, Hq, Hkv, N, d = 1, 24, 2, 700, 128
    K, V = workload(B, Hkv, N, d, seed=9)
    ch = SP.select_outlier_channels(host(K[0, 0, :64]), 32)
    kq = api.SplitQuantizer(d, ch, 3, 2, "mse", seed_rot=21, device=DEV)
    vq = api.SplitQuantizer(d, ch, 3, 2, "prod", seed_rot=23, seed_qjl=24, device=DEV)
    kc, vc = api.encode_split(kq, K.to(DEV)), api.encode_split(vq, V.to(DEV))
    q = torch.randn((B, Hq, d), generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    out = host(api.DecodeAttentionSplit(kq, vq, B, Hq, Hkv, N, device=DEV)(q.to(DEV), kc, vc))
    okq = SP.SplitQuantizer(d, ch, 3, 2, "mse", seed_rot=21)
    ovq = SP.SplitQuantizer(d, ch, 3, 2, "prod", seed_rot=23, seed_qjl=24)
    qh = host(q)
    for h in range(Hkv):
        ke = SP.encode(okq, host(K[0, h]), aux=False)
        ve = SP.encode(ovq, host(V[0, h]), aux=False)
        for hq in range(h * 12, (h + 1) * 12):
            ref = SP.decode_attention(okq, ovq, qh[0, hq], ke, ve, dtype=np.float32)
            assert rel_err(out[0, hq], ref) <= 2e-3, hq
