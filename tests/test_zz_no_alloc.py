"""tq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (e.g. a plugin running inside an engine that owns
all device allocations).  It uses the library's fixed scratch array instead
of a caller workspace; its results must equal tq_decode_attention's.

This file is collected last, so a run that stops at the first failure has
run every other test before it; it also passes on its own in a fresh
process."""

import ctypes
import math

import numpy as np
import pytest
import torch

from kv_cache_vector_13_b200 import _lib as L
from kv_cache_vector_13_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3  # the attention tolerance of the other decode tests


def _noalloc(kq, vq, q, kc, vc, out, scores=None, seq_lens=None):
    kv, vv = kc.view(), vc.view()
    B, Hq, _ = q.shape
    _, Hkv, N = kc.shape
    st = L.lib().tq_decode_attention_noalloc(
        ctypes.byref(kq.c_struct()), ctypes.byref(vq.c_struct()), q.data_ptr(), L.TQ_BF16, B, Hq, Hkv, N,
        None if seq_lens is None else seq_lens.data_ptr(), ctypes.byref(kv), ctypes.byref(vv),
        1.0 / math.sqrt(q.shape[-1]), out.data_ptr(), None if scores is None else scores.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    return st


def _problem(seed, B=2, Hq=8, Hkv=2, N=5000, d=128):
    g = torch.Generator(device=DEV).manual_seed(seed)
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV).to(torch.bfloat16)
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV).to(torch.bfloat16)
    kq = api.Quantizer(d, 3, "prod", seed_rot=5, seed_qjl=6, device=DEV)
    vq = api.Quantizer(d, 4, "mse", seed_rot=7, device=DEV)
    return g, kq, vq, api.encode(kq, K), api.encode(vq, V)


def test_noalloc_matches_workspace_entry_point_twice():
    # both entry points run the same kernels on the same data with a fixed
    # merge order, so the outputs agree bit for bit (and so within the 2e-3
    # attention tolerance of the other decode tests)
    B, Hq, d = 2, 8, 128
    g, kq, vq, kc, vc = _problem(11)
    for call in range(2):
        q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
        ref = api.decode_attention(kq, vq, q, kc, vc)
        out = torch.full((B, Hq, d), float("nan"), device=DEV)
        assert _noalloc(kq, vq, q, kc, vc, out) == L.TQ_OK, L.last_error()
        torch.cuda.synchronize()
        o, r = out.cpu().numpy(), ref.cpu().numpy()
        err = (np.abs(o - r).max(axis=-1) / np.abs(r).max(axis=-1)).max()
        assert err <= TOL, f"call {call}: {err:.2e}"
        assert torch.equal(out, ref), f"call {call}: outputs differ"


def test_noalloc_ragged_lengths_and_scores_twice():
    # per-batch lengths and the scores output through the static scratch,
    # twice in a row (the second call starts from the first call's scratch)
    B, Hq, N, d = 2, 8, 5000, 128
    g, kq, vq, kc, vc = _problem(12)
    lens = torch.tensor([N - 123, 777], dtype=torch.int32, device=DEV)
    for call in range(2):
        q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
        s_ref = torch.full((B, Hq, N), -3.0, device=DEV)
        ref = api.decode_attention(kq, vq, q, kc, vc, seq_lens=lens, scores=s_ref)
        out = torch.full((B, Hq, d), float("nan"), device=DEV)
        s_got = torch.full((B, Hq, N), -3.0, device=DEV)
        assert _noalloc(kq, vq, q, kc, vc, out, scores=s_got, seq_lens=lens) == L.TQ_OK, L.last_error()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: outputs differ"
        assert torch.equal(s_got, s_ref), f"call {call}: scores differ"


def test_noalloc_rejects_problems_beyond_its_scratch():
    # real (small) device buffers throughout, so that a regression of the
    # size check shows up as a wrong status rather than as a launch on
    # addresses that do not exist
    B, Hq, Hkv, N, d = 4096, 64, 8, 16, 128
    kq = api.Quantizer(d, 4, "mse", device=DEV)
    vq = api.Quantizer(d, 4, "mse", device=DEV)
    need = api.decode_workspace_bytes(B, Hq, Hkv, N, d)
    assert need > L.TQ_NOALLOC_SCRATCH_BYTES
    kc, vc = api.empty_cache(kq, B, Hkv, N, DEV), api.empty_cache(vq, B, Hkv, N, DEV)
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros((B, Hq, d), device=DEV)
    assert _noalloc(kq, vq, q, kc, vc, out) == L.TQ_EWORKSPACE
    assert "static scratch" in L.last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0
