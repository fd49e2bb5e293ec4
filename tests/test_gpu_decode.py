"""GPU parity of tq_decode_attention against the fp32 oracle.

Tolerance: max |o - o_ref| / max |o_ref| <= 2e-3 per (batch, query head),
against the oracle evaluated in fp32 on the oracle's own encoding of the
same inputs (codes are bit-exact, so both see the same cache)."""

import math

import numpy as np
import pytest
import torch

from kv_cache_vector_13_b200 import _lib as L
from kv_cache_vector_13_b200 import api, inputs
from oracle import attention as OA
from oracle import metrics as OM
from oracle import quantizer as OQ

from helpers import (compare_records, compare_slice_records, flat_host, host, oracle_attention,
                     oracle_cache_slices, oracle_twin, rel_err)

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def run_case(B, Hq, Hkv, N, kspec, vspec, seed=0, seq_lens=None, kv_scale=1.0, heads=None, scores=False, d=128,
             rotation=("hadamard", "hadamard"), zero_q_heads=()):
    g = torch.Generator(device=DEV).manual_seed(seed)
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV) * kv_scale
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
    for h in zero_q_heads:
        q[:, h] = 0
    kq = api.Quantizer(d, kspec[0], kspec[1], seed_rot=seed + 1, seed_qjl=seed + 2, device=DEV, rotation=rotation[0])
    vq = api.Quantizer(d, vspec[0], vspec[1], seed_rot=seed + 3, seed_qjl=seed + 4, device=DEV,
                       rotation=rotation[1])
    kc, vc = api.encode(kq, K), api.encode(vq, V)
    sl = None if seq_lens is None else torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
    sc = torch.full((B, Hq, N), float("nan"), device=DEV) if scores else None
    out = host(api.decode_attention(kq, vq, q, kc, vc, seq_lens=sl, scores=sc))
    okq, ovq = oracle_twin(kq), oracle_twin(vq)
    okc, _ = oracle_cache_slices(okq, host(K))
    ovc, _ = oracle_cache_slices(ovq, host(V))
    qh = host(q)
    todo = heads or [(b, h) for b in range(B) for h in range(Hq)]
    for (b, h) in todo:
        L = N if seq_lens is None else seq_lens[b]
        if L == 0:
            assert np.all(out[b, h] == 0)
            continue
        kcs = {k: v[b:b + 1, :, :L] for k, v in okc.items()}
        vcs = {k: v[b:b + 1, :, :L] for k, v in ovc.items()}
        res = OA.decode_attention(okq, ovq, qh[b:b + 1].astype(np.float32), kcs, vcs, dtype=np.float32,
                                  heads=[(0, h)], return_scores=scores)
        ref = res[0] if scores else res
        e = rel_err(out[b, h], ref[0, h])
        assert e <= TOL, f"(b={b}, h={h}, L={L}) rel err {e:.2e}"
        if scores:
            s_gpu = host(sc)[b, h, :L]
            s_ref = res[1][0, h]
            np.testing.assert_allclose(s_gpu, s_ref, rtol=2e-3, atol=2e-3 * np.abs(s_ref).max())
    return out


@pytest.mark.parametrize("kspec,vspec", [((4, "mse"), (4, "mse")), ((3, "mse"), (3, "mse")),
                                         ((3, "prod"), (3, "mse")), ((4, "prod"), (4, "mse")),
                                         ((2, "mse"), (2, "mse")), ((1, "mse"), (1, "mse")),
                                         ((2, "prod"), (1, "mse")), ((1, "prod"), (4, "mse"))])
def test_decode_small_grid(kspec, vspec):
    run_case(2, 8, 2, 1000 + 29, kspec, vspec, seed=10 * kspec[0] + vspec[0] + (100 if kspec[1] == 'prod' else 0), scores=True)


@pytest.mark.parametrize("N", [1, 2, 31, 32, 33, 63, 64, 65, 257, 4097])
def test_decode_ragged_lengths(N):
    run_case(1, 4, 1, N, (4, "mse"), (4, "mse"), seed=N)


@pytest.mark.parametrize("g", [1, 2, 3, 4, 6, 8, 16])
def test_decode_gqa_group_sizes(g):
    run_case(1, 2 * g, 2, 700, (3, "prod"), (3, "mse"), seed=g)


@pytest.mark.parametrize("Hq,kspec", [(8, (3, "prod")), (16, (4, "prod")), (8, (1, "prod"))])
def test_decode_zero_query_heads(Hq, kspec):
    # a zero query: S q' = 0 (its int8 digit scale falls back to 1), every
    # score is 0 and the softmax is uniform
    run_case(1, Hq, 2, 513, kspec, (3, "mse"), seed=40 + Hq, zero_q_heads=(0, 5), scores=True)


def test_decode_per_batch_lengths_including_empty():
    run_case(4, 4, 2, 900, (4, "mse"), (3, "mse"), seed=7, seq_lens=[900, 0, 1, 333])


def test_decode_large_logits():
    # sharp softmax: keys scaled so that a few tokens dominate
    run_case(1, 8, 1, 2048, (4, "prod"), (4, "mse"), seed=9, kv_scale=6.0)


def test_decode_config1_scores_shared_cache():
    # one head, d=128, N=4096 keys from seed 0, 16 queries from seed 1, mse b=3:
    # the 16 queries are a batch of 16 that shares one cache (stride_b = 0)
    d, N = 128, 4096
    x = inputs.vectors(N, d, seed=0, device=DEV)
    qs = inputs.vectors(16, d, seed=1, device=DEV)
    kq = api.Quantizer(d, 3, "mse", seed_rot=0, device=DEV)
    vq = api.Quantizer(d, 3, "mse", seed_rot=1, device=DEV)
    kc = api.encode(kq, x)
    vc = api.encode(vq, x)
    shared_k = api.PackedCache(kc.codes.expand(16, 1, N, -1), kc.norms.expand(16, 1, N))
    shared_v = api.PackedCache(vc.codes.expand(16, 1, N, -1), vc.norms.expand(16, 1, N))
    sc = torch.empty((16, 1, N), device=DEV)
    out = host(api.decode_attention(kq, vq, qs[:, None, :].contiguous(), shared_k, shared_v, scores=sc))
    okq, ovq = oracle_twin(kq), oracle_twin(vq)
    okc, _ = oracle_cache_slices(okq, host(x)[None, None])
    ovc, _ = oracle_cache_slices(ovq, host(x)[None, None])
    qh = host(qs)
    for i in range(16):
        o, s = OA.decode_attention(okq, ovq, qh[i][None, None], okc, ovc, dtype=np.float32, return_scores=True)
        assert rel_err(out[i, 0], o[0, 0]) <= TOL
        np.testing.assert_allclose(host(sc)[i, 0], s[0, 0], rtol=1e-3, atol=1e-3 * np.abs(s).max())


def test_decode_config2_full_size():
    # Llama-3.1-8B-shaped layer: B=1, 32 q heads, 8 kv heads, N=32768, mse b=4
    N = 32768
    K, V = inputs.llama8b_kv(N=N, device=DEV)
    q = inputs.queries(1, 32, device=DEV)
    kq = api.Quantizer(128, 4, "mse", seed_rot=10, device=DEV)
    vq = api.Quantizer(128, 4, "mse", seed_rot=11, device=DEV)
    kc, vc = api.encode(kq, K), api.encode(vq, V)
    out = host(api.decode_attention(kq, vq, q, kc, vc))
    okq, ovq = oracle_twin(kq), oracle_twin(vq)
    okc, kenc = oracle_cache_slices(okq, host(K))
    ovc, venc = oracle_cache_slices(ovq, host(V))
    # the packed records of all 8 KV heads, bit for bit
    compare_records(kq, okq, kenc, flat_host(kc))
    compare_records(vq, ovq, venc, flat_host(vc))
    ref = oracle_attention(okq, ovq, host(q), okc, ovc)
    e = rel_err(out, ref)
    assert e.max() <= TOL, e.max()


def sampled_decode(K, V, q, kq, vq, kv_heads):
    """Decode the whole cache on the GPU; for the sampled (batch, kv head)
    slices, compare every packed record with the oracle's (codes, norms and
    residual norms bit for bit, QJL signs up to the fp32 band, at most a
    1e-6 fraction of them) and the attention outputs of the slice's query
    heads with the fp32 oracle."""
    kc, vc = api.encode(kq, K), api.encode(vq, V)
    out = host(api.decode_attention(kq, vq, q, kc, vc))
    okq, ovq = oracle_twin(kq), oracle_twin(vq)
    Hq, Hkv, N, d = q.shape[1], K.shape[1], K.shape[2], K.shape[3]
    g = Hq // Hkv
    worst = 0.0
    for (b, h) in kv_heads:
        nk = compare_slice_records(kq, okq, host(K[b, h]), kc, b, h)
        assert nk <= max(2, 1e-6 * N * d), f"slice ({b}, {h}): {nk} QJL bits differ"
        compare_slice_records(vq, ovq, host(V[b, h]), vc, b, h)
        okc, _ = oracle_cache_slices(okq, host(K[b:b + 1, h:h + 1]))
        ovc, _ = oracle_cache_slices(ovq, host(V[b:b + 1, h:h + 1]))
        qb = host(q[b:b + 1, h * g:(h + 1) * g])
        ref = oracle_attention(okq, ovq, qb, okc, ovc)
        e = rel_err(out[b, h * g:(h + 1) * g], ref[0]).max()
        worst = max(worst, e)
        assert e <= TOL, (b, h, e)
    return worst


def test_decode_config3_sampled():
    # batch 16, 32/8 heads, N=131072, 2% outlier channels x8; K prod b=3, V mse b=3
    K, V = inputs.outlier_kv(N=131072, B=16, device=DEV)
    q = inputs.queries(16, 32, device=DEV)
    kq = api.Quantizer(128, 3, "prod", seed_rot=20, seed_qjl=21, device=DEV)
    vq = api.Quantizer(128, 3, "mse", seed_rot=22, device=DEV)
    sampled_decode(K, V, q, kq, vq, [(0, 0), (15, 7), (9, 3)])


def test_decode_config5_sampled():
    # 70B-shaped long context: B=1, 64/8 heads, N=2^20, Student-t values
    K, V = inputs.student_kv(N=1 << 20, device=DEV)
    q = inputs.queries(1, 64, device=DEV)
    kq = api.Quantizer(128, 4, "prod", seed_rot=30, seed_qjl=31, device=DEV)
    vq = api.Quantizer(128, 4, "mse", seed_rot=32, device=DEV)
    sampled_decode(K, V, q, kq, vq, [(0, 0), (0, 5)])


def test_decode_config1_codes_norms_and_mse():
    # config 1's remaining outputs: the packed codes and norms of the 4096
    # keys (bit for bit), and the MSE on unit-normalised vectors, measured
    # through the GPU encode + dequant and equal to the oracle's
    d, N = 128, 4096
    x = inputs.vectors(N, d, seed=0, device=DEV)
    kq = api.Quantizer(d, 3, "mse", seed_rot=0, device=DEV)
    kc = api.encode(kq, x)
    okq = oracle_twin(kq)
    enc = OQ.encode(okq, host(x))
    compare_records(kq, okq, enc, flat_host(kc))
    xu = x / x.norm(dim=1, keepdim=True)
    cu = api.encode(kq, xu)
    xh = api.dequant(kq, cu)[0, 0].double()
    mse_gpu = float(((xu.double() - xh) ** 2).sum(dim=1).mean())
    mse_ref, se = OM.mse(okq, host(xu))
    compare_records(kq, okq, OQ.encode(okq, host(xu)), flat_host(cu))
    assert abs(mse_gpu - mse_ref) <= 1e-5 * mse_ref, (mse_gpu, mse_ref)
    # the sphere value for b = 3 at d = 128 is 0.0340, within sampling error
    assert abs(mse_gpu - 0.0340) <= 4 * se + 5e-4, (mse_gpu, se)


@pytest.mark.parametrize("kspec", [(4, "mse"), (3, "prod")])
def test_decode_token_major_cache(kspec):
    # a [B, N, Hkv]-major cache (stride_n = Hkv records): the kernel's general
    # record addressing; the cache is written by tq_encode through the same
    # strided view
    B, Hq, Hkv, N, d = 2, 8, 2, 777, 128
    g = torch.Generator(device=DEV).manual_seed(41)
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
    kq = api.Quantizer(d, kspec[0], kspec[1], seed_rot=42, seed_qjl=43, device=DEV)
    vq = api.Quantizer(d, 3, "mse", seed_rot=44, device=DEV)

    def token_major(qz):
        def arr(w, dt):
            t = torch.empty((B, N, Hkv, w), dtype=dt, device=DEV).permute(0, 2, 1, 3)
            return t if w > 1 else t[..., 0]
        return api.PackedCache(arr(qz.code_bytes, torch.uint8) if qz.bm else None, arr(1, torch.float32),
                               arr(qz.qjl_bytes, torch.uint8) if qz.prod else None,
                               arr(1, torch.float32) if qz.prod else None)

    kc, vc = token_major(kq), token_major(vq)
    assert kc.view().stride_n == Hkv and kc.view().stride_h == 1
    api.encode(kq, K, out=kc)
    api.encode(vq, V, out=vc)
    sl = torch.tensor([N, N - 300], dtype=torch.int32, device=DEV)
    out = host(api.decode_attention(kq, vq, q, kc, vc, seq_lens=sl))
    okq, ovq = oracle_twin(kq), oracle_twin(vq)
    okc, _ = oracle_cache_slices(okq, host(K))
    ovc, _ = oracle_cache_slices(ovq, host(V))
    for b in range(B):
        L = int(sl[b])
        kcs = {k: v[b:b + 1, :, :L] for k, v in okc.items()}
        vcs = {k: v[b:b + 1, :, :L] for k, v in ovc.items()}
        ref = oracle_attention(okq, ovq, host(q)[b:b + 1], kcs, vcs)
        e = rel_err(out[b], ref[0]).max()
        assert e <= TOL, (b, e)


def test_decode_zero_norm_rows():
    # zero key and value vectors: n = 0, so the key's score is 0 and the
    # value's weight p_j n_j is 0 (log2 n = -inf inside the kernel)
    B, Hq, Hkv, N, d = 1, 8, 2, 1500, 128
    g = torch.Generator(device=DEV).manual_seed(51)
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    K[:, :, 3::11] = 0.0
    V[:, :, ::7] = 0.0
    V[:, 1, :64] = 0.0  # a whole chunk of zero values on one head
    q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
    kq = api.Quantizer(d, 4, "prod", seed_rot=52, seed_qjl=53, device=DEV)
    vq = api.Quantizer(d, 4, "mse", seed_rot=54, device=DEV)
    kc, vc = api.encode(kq, K), api.encode(vq, V)
    assert int((vc.norms == 0).sum()) > 0
    out = host(api.decode_attention(kq, vq, q, kc, vc))
    assert np.all(np.isfinite(out))
    okq, ovq = oracle_twin(kq), oracle_twin(vq)
    okc, _ = oracle_cache_slices(okq, host(K))
    ovc, _ = oracle_cache_slices(ovq, host(V))
    ref = oracle_attention(okq, ovq, host(q), okc, ovc)
    assert rel_err(out, ref).max() <= TOL


def test_decode_repeated_calls_reuse_workspace():
    # the per-unit arrival counters live in the workspace and are re-armed by
    # every call: three calls through one workspace give identical outputs
    g = torch.Generator(device=DEV).manual_seed(3)
    K = torch.randn((2, 2, 3000, 128), generator=g, device=DEV)
    V = torch.randn((2, 2, 3000, 128), generator=g, device=DEV)
    q = torch.randn((2, 8, 128), generator=g, device=DEV).to(torch.bfloat16)
    kq = api.Quantizer(128, 4, "mse", seed_rot=1, device=DEV)
    vq = api.Quantizer(128, 4, "mse", seed_rot=2, device=DEV)
    kc, vc = api.encode(kq, K), api.encode(vq, V)
    op = api.DecodeAttention(kq, vq, 2, 8, 2, 3000, device=DEV)
    outs = [op(q, kc, vc).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    ref = api.decode_attention(kq, vq, q, kc, vc)
    assert torch.equal(outs[0], ref)


@pytest.mark.parametrize("Hq,Hkv,kspec,vspec,dtype", [
    (8, 2, (4, "mse"), (4, "mse"), torch.bfloat16),
    (8, 2, (3, "prod"), (3, "mse"), torch.float32),
    (16, 2, (4, "prod"), (2, "mse"), torch.float16),
])
def test_append_decode_matches_separate_calls(Hq, Hkv, kspec, vspec, dtype):
    # tq_append_decode_attention = tq_encode of the new K and V into the tail
    # records + tq_decode_attention: same tail records and the same output
    # bits, over two steps in a row through one workspace
    B, N, d = 2, 1000, 128
    g = torch.Generator(device=DEV).manual_seed(71)
    kq = api.Quantizer(d, kspec[0], kspec[1], seed_rot=72, seed_qjl=73, device=DEV)
    vq = api.Quantizer(d, vspec[0], vspec[1], seed_rot=74, device=DEV)
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV).to(dtype)
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV).to(dtype)
    ka, va = api.encode(kq, K), api.encode(vq, V)
    kb = api.PackedCache(*(None if t is None else t.clone() for t in (ka.codes, ka.norms, ka.qjl, ka.rnorms)))
    vb = api.PackedCache(*(None if t is None else t.clone() for t in (va.codes, va.norms, va.qjl, va.rnorms)))

    def tail(c, n):
        return api.PackedCache(*(None if t is None else t[:, :, n:n + 1] for t in (c.codes, c.norms, c.qjl, c.rnorms)))

    op = api.DecodeAttention(kq, vq, B, Hq, Hkv, N, device=DEV)
    okq, ovq = oracle_twin(kq), oracle_twin(vq)
    Kh, Vh = host(K), host(V)
    for step, n in enumerate((N - 1, N - 2)):
        q = torch.randn((B, Hq, d), generator=g, device=DEV).to(dtype)
        k_new = torch.randn((B, Hkv, d), generator=g, device=DEV).to(dtype)
        v_new = torch.randn((B, Hkv, d), generator=g, device=DEV).to(dtype)
        api.encode(kq, k_new[:, :, None], out=tail(ka, n))
        api.encode(vq, v_new[:, :, None], out=tail(va, n))
        ref = api.decode_attention(kq, vq, q, ka, va)
        got = op.append_step(q, k_new, v_new, tail(kb, n), tail(vb, n), kb, vb).clone()
        torch.cuda.synchronize()
        for a_, b_ in ((ka, kb), (va, vb)):
            for t1, t2 in zip((a_.codes, a_.norms, a_.qjl, a_.rnorms), (b_.codes, b_.norms, b_.qjl, b_.rnorms)):
                if t1 is not None:
                    assert torch.equal(t1, t2), f"step {step}: cache records differ"
        assert torch.equal(ref, got), f"step {step}: max diff {(ref - got).abs().max().item()}"
        # and the fused step against the oracle: the cache with the new
        # token written at n, encoded and attended by the oracle
        Kh[:, :, n], Vh[:, :, n] = host(k_new), host(v_new)
        okc, _ = oracle_cache_slices(okq, Kh)
        ovc, _ = oracle_cache_slices(ovq, Vh)
        e = rel_err(host(got), oracle_attention(okq, ovq, host(q), okc, ovc)).max()
        assert e <= TOL, f"step {step}: fused step vs oracle {e:.2e}"


def test_append_decode_rejects_bad_tail_before_any_launch():
    # a misaligned new-token stride is refused with TQ_EINVAL and nothing runs
    B, Hq, Hkv, N, d = 1, 4, 1, 64, 128
    kq = api.Quantizer(d, 4, "mse", seed_rot=1, device=DEV)
    vq = api.Quantizer(d, 4, "mse", seed_rot=2, device=DEV)
    kc, vc = api.empty_cache(kq, B, Hkv, N, DEV), api.empty_cache(vq, B, Hkv, N, DEV)
    op = api.DecodeAttention(kq, vq, B, Hq, Hkv, N, device=DEV)
    q = torch.zeros((B, Hq, d), device=DEV)
    buf = torch.zeros((B, Hkv, d + 1), device=DEV)  # row stride d + 1 floats: not a 16-byte multiple
    k_new = buf[:, :, :d]
    tk = api.PackedCache(kc.codes[:, :, -1:], kc.norms[:, :, -1:])
    tv = api.PackedCache(vc.codes[:, :, -1:], vc.norms[:, :, -1:])
    with pytest.raises(L.TqError) as e:
        op.append_step(q, k_new, k_new, tk, tv, kc, vc)
    assert e.value.status == L.TQ_EINVAL


def test_append_decode_with_batch_lengths_and_scores():
    # ragged per-batch lengths and the scores output through the fused step:
    # identical to the separate calls (tail at a position every batch attends)
    B, Hq, Hkv, N, d = 2, 8, 2, 700, 128
    g = torch.Generator(device=DEV).manual_seed(81)
    kq = api.Quantizer(d, 3, "prod", seed_rot=82, seed_qjl=83, device=DEV)
    vq = api.Quantizer(d, 4, "mse", seed_rot=84, device=DEV)
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV).to(torch.bfloat16)
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV).to(torch.bfloat16)
    ka, va = api.encode(kq, K), api.encode(vq, V)
    kb = api.PackedCache(*(None if t is None else t.clone() for t in (ka.codes, ka.norms, ka.qjl, ka.rnorms)))
    vb = api.PackedCache(*(None if t is None else t.clone() for t in (va.codes, va.norms, va.qjl, va.rnorms)))
    lens = torch.tensor([N, N - 37], dtype=torch.int32, device=DEV)
    n = N - 40

    def tail(c):
        return api.PackedCache(*(None if t is None else t[:, :, n:n + 1] for t in (c.codes, c.norms, c.qjl, c.rnorms)))

    q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
    k_new = torch.randn((B, Hkv, d), generator=g, device=DEV).to(torch.bfloat16)
    v_new = torch.randn((B, Hkv, d), generator=g, device=DEV).to(torch.bfloat16)
    api.encode(kq, k_new[:, :, None], out=tail(ka))
    api.encode(vq, v_new[:, :, None], out=tail(va))
    s_ref = torch.full((B, Hq, N), -7.0, device=DEV)
    ref = api.decode_attention(kq, vq, q, ka, va, seq_lens=lens, scores=s_ref)
    s_got = torch.full((B, Hq, N), -7.0, device=DEV)
    op = api.DecodeAttention(kq, vq, B, Hq, Hkv, N, device=DEV)
    got = op.append_step(q, k_new, v_new, tail(kb), tail(vb), kb, vb, seq_lens=lens, scores=s_got).clone()
    torch.cuda.synchronize()
    assert torch.equal(ref, got)
    assert torch.equal(s_ref, s_got)


# The CUDA-core path: d other than 128, prod values, dense rotations of any
# d; ragged lengths (one batch empty), scores, a GQA group of 12 (two head
# groups of a block) and a long enough cache for several sequence splits.
@pytest.mark.parametrize("d,kspec,vspec,rotation,g", [
    (64, (3, "prod"), (3, "mse"), ("hadamard", "hadamard"), 4),
    (256, (4, "mse"), (3, "prod"), ("hadamard", "hadamard"), 4),
    (128, (3, "prod"), (3, "prod"), ("hadamard", "hadamard"), 12),
    (128, (2, "mse"), (2, "prod"), ("dense", "dense"), 4),
    (200, (3, "mse"), (4, "mse"), ("dense", "dense"), 2),
    (64, (1, "prod"), (1, "prod"), ("hadamard", "dense"), 1),
    # the smallest dense d (one-word records, 64 token classes) and a d whose
    # code and sign records are not whole words (byte-wise staging)
    (8, (2, "mse"), (3, "mse"), ("dense", "dense"), 4),
    (40, (4, "prod"), (2, "prod"), ("dense", "dense"), 8),
])
def test_decode_cuda_core_path(d, kspec, vspec, rotation, g):
    Hkv = 2
    run_case(3, g * Hkv, Hkv, 1500, kspec, vspec, seed=d + 7 * g + kspec[0], seq_lens=[1500, 0, 613],
             scores=True, d=d, rotation=rotation)


def test_decode_cuda_core_path_long_cache():
    # one (batch, kv head) over 40000 tokens: the sequence split across blocks
    out = run_case(1, 4, 1, 40000, (4, "prod"), (4, "prod"), seed=77, d=256, kv_scale=3.0)
    assert np.all(np.isfinite(out))



@pytest.fixture
def bulk_staged_feed():
    prev = api.set_decode_feed(True)
    yield
    api.set_decode_feed(prev)


@pytest.mark.parametrize("kspec,vspec,Hq", [((3, "prod"), (3, "mse"), 32), ((4, "mse"), (4, "mse"), 32),
                                            ((4, "prod"), (4, "mse"), 64), ((2, "mse"), (2, "mse"), 16)])
def test_decode_bulk_staged_feed_matches_oracle(bulk_staged_feed, kspec, vspec, Hq):
    # the bulk-copy ring feed (shared-memory slots filled by cp.async.bulk,
    # mbarrier waits) on unit-stride caches with 16-byte aligned norm rows:
    # <= 4 and 8 query heads per kv head, prod and mse keys, a ragged batch
    B, Hkv, N = 2, 8, 1000
    heads = [(0, 0), (0, Hq - 1), (1, 1), (1, Hq // 2)]
    out = run_case(B, Hq, Hkv, N, kspec, vspec, seed=21, seq_lens=[N, 613], heads=heads)
    api.check()  # no bounded wait gave up, no layout fault
    assert torch.isfinite(torch.as_tensor(out)).all()


def test_decode_bulk_staged_feed_agrees_with_register_feed(bulk_staged_feed):
    # the same call through both feeds: equal up to the summation order of
    # the warps' partials
    g = torch.Generator(device=DEV).manual_seed(5)
    B, Hq, Hkv, N, d = 3, 32, 8, 2048, 128
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV)
    q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
    kq = api.Quantizer(d, 3, "prod", seed_rot=1, seed_qjl=2, device=DEV)
    vq = api.Quantizer(d, 3, "mse", seed_rot=3, device=DEV)
    kc, vc = api.encode(kq, K), api.encode(vq, V)
    staged = api.decode_attention(kq, vq, q, kc, vc)
    api.check()
    api.set_decode_feed(False)
    regs = api.decode_attention(kq, vq, q, kc, vc)
    e = ((staged - regs).abs().amax(dim=-1) / regs.abs().amax(dim=-1)).max().item()
    assert e <= 1e-4, e
