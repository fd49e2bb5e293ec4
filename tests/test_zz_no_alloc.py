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


def _noalloc(kq, vq, q, kc, vc, out, scores=None):
    kv, vv = kc.view(), vc.view()
    B, Hq, _ = q.shape
    _, Hkv, N = kc.shape
    st = L.lib().tq_decode_attention_noalloc(
        ctypes.byref(kq.c_struct()), ctypes.byref(vq.c_struct()), q.data_ptr(), L.TQ_BF16, B, Hq, Hkv, N, None,
        ctypes.byref(kv), ctypes.byref(vv), 1.0 / math.sqrt(q.shape[-1]), out.data_ptr(),
        None if scores is None else scores.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return st


def test_noalloc_matches_workspace_entry_point_twice():
    g = torch.Generator(device=DEV).manual_seed(11)
    B, Hq, Hkv, N, d = 2, 8, 2, 5000, 128
    K = torch.randn((B, Hkv, N, d), generator=g, device=DEV).to(torch.bfloat16)
    V = torch.randn((B, Hkv, N, d), generator=g, device=DEV).to(torch.bfloat16)
    kq = api.Quantizer(d, 3, "prod", seed_rot=5, seed_qjl=6, device=DEV)
    vq = api.Quantizer(d, 4, "mse", seed_rot=7, device=DEV)
    kc, vc = api.encode(kq, K), api.encode(vq, V)
    for call in range(2):
        q = torch.randn((B, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
        ref = api.decode_attention(kq, vq, q, kc, vc)
        out = torch.full((B, Hq, d), float("nan"), device=DEV)
        assert _noalloc(kq, vq, q, kc, vc, out) == L.TQ_OK, L.last_error()
        torch.cuda.synchronize()
        o, r = out.cpu().numpy(), ref.cpu().numpy()
        err = (np.abs(o - r).max(axis=-1) / np.abs(r).max(axis=-1)).max()
        assert err <= TOL, f"call {call}: {err:.2e}"


def test_noalloc_rejects_problems_beyond_its_scratch():
    kq = api.Quantizer(128, 4, "mse", device=DEV)
    vq = api.Quantizer(128, 4, "mse", device=DEV)
    # B * Hq * d * 8 bytes of rotated queries alone exceed the scratch
    B, Hq, Hkv = 4096, 64, 8
    need = api.decode_workspace_bytes(B, Hq, Hkv, 16, 128)
    assert need > L.TQ_NOALLOC_SCRATCH_BYTES
    fake = L.TqCacheView(0x10000, None, 0x10000, None, 0, 0, 1)
    st = L.lib().tq_decode_attention_noalloc(
        ctypes.byref(kq.c_struct()), ctypes.byref(vq.c_struct()), 0x10000, L.TQ_BF16, B, Hq, Hkv, 16, None,
        ctypes.byref(fake), ctypes.byref(fake), 0.1, 0x10000, None, None)
    assert st == L.TQ_EWORKSPACE
    assert "static scratch" in L.last_error()
