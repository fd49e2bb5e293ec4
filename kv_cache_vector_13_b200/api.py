"""Thin torch binding of the TurboQuant C ABI (argument marshalling only).

Every step of encode, dequant and decode attention runs in the CUDA kernels
of libtq_b200.so; torch supplies device memory, strides and the current
stream.  The names follow the C ABI (include/tq.h).
"""

import ctypes
import math
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import _lib as L

_DTYPES = {torch.float32: L.TQ_F32, torch.bfloat16: L.TQ_BF16, torch.float16: L.TQ_F16}


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


# ------------------------------------------------------------- host calls

def make_codebook(d: int, bits_mse: int, dist: str = "gauss"):
    """(centroids, thresholds) as numpy fp32 arrays from tq_make_codebook."""
    K = 1 << bits_mse
    c = (ctypes.c_float * K)()
    t = (ctypes.c_float * max(K - 1, 1))()
    L.check(L.lib().tq_make_codebook(d, bits_mse, L.TQ_CB_BETA if dist == "beta" else L.TQ_CB_GAUSS, c, t))
    return np.frombuffer(c, np.float32).copy(), np.frombuffer(t, np.float32)[: K - 1].copy()


def make_signs(seed: int, d: int) -> np.ndarray:
    s = np.empty(d, np.int8)
    L.check(L.lib().tq_make_signs(seed, d, s.ctypes.data))
    return s


def make_qjl(seed: int, d: int) -> np.ndarray:
    S = np.empty((d, d), np.float32)
    L.check(L.lib().tq_make_qjl(seed, d, S.ctypes.data_as(ctypes.POINTER(ctypes.c_float))))
    return S


def make_rotation(seed: int, d: int) -> np.ndarray:
    """Dense Haar rotation Pi (tq_make_rotation), numpy fp32 [d, d]."""
    R = np.empty((d, d), np.float32)
    L.check(L.lib().tq_make_rotation(seed, d, R.ctypes.data_as(ctypes.POINTER(ctypes.c_float))))
    return R


def code_bytes(d: int, bits: int, variant: str) -> int:
    return int(L.lib().tq_code_bytes(d, bits, L.TQ_PROD if variant == "prod" else L.TQ_MSE))


def qjl_bytes(d: int, variant: str) -> int:
    return int(L.lib().tq_qjl_bytes(d, L.TQ_PROD if variant == "prod" else L.TQ_MSE))


# ------------------------------------------------------------ quantizer

class Quantizer:
    """Device-resident parameters of one TurboQuant quantizer."""

    def __init__(self, d: int, bits: int, variant: str = "mse", seed_rot: int = 0,
                 seed_qjl: int = 1, dist: str = "gauss", device="cuda", rotation: str = "hadamard",
                 channels: Optional[torch.Tensor] = None):
        assert variant in ("mse", "prod") and rotation in ("hadamard", "dense")
        self.d, self.bits, self.variant = d, bits, variant
        self.seed_rot, self.seed_qjl, self.dist, self.rotation = seed_rot, seed_qjl, dist, rotation
        self.bm = bits - 1 if variant == "prod" else bits
        dev = torch.device(device)
        if self.bm > 0:
            c, t = make_codebook(d, self.bm, dist)
            self.centroids = torch.from_numpy(c).to(dev)
            self.thresholds = torch.from_numpy(t).to(dev) if t.size else torch.zeros(1, device=dev)
        else:
            self.centroids = self.thresholds = None
        self.signs = torch.from_numpy(make_signs(seed_rot, d)).to(dev)
        self.S = torch.from_numpy(make_qjl(seed_qjl, d)).to(dev) if variant == "prod" else None
        self.rot = torch.from_numpy(make_rotation(seed_rot, d)).to(dev) if rotation == "dense" else None
        self.channels = None if channels is None else channels.to(device=dev, dtype=torch.int32).contiguous()
        self._c = L.TqQuantizer(d, bits, L.TQ_PROD if variant == "prod" else L.TQ_MSE,
                                L.TQ_ROT_DENSE if rotation == "dense" else L.TQ_ROT_HADAMARD,
                                _ptr(self.centroids), _ptr(self.thresholds), _ptr(self.signs), _ptr(self.S),
                                _ptr(self.rot), _ptr(self.channels))

    @property
    def prod(self) -> bool:
        return self.variant == "prod"

    @property
    def code_bytes(self) -> int:
        return self.d * self.bm // 8

    @property
    def qjl_bytes(self) -> int:
        return self.d // 8 if self.prod else 0

    @property
    def record_bytes(self) -> int:
        """Stored bytes per vector: codes + sketch + fp32 norms."""
        return self.code_bytes + self.qjl_bytes + 4 + (4 if self.prod else 0)

    def c_struct(self) -> L.TqQuantizer:
        return self._c


@dataclass
class PackedCache:
    """Packed records shaped [B, H, N, ...] (any strides over B, H, N)."""
    codes: Optional[torch.Tensor]
    norms: torch.Tensor
    qjl: Optional[torch.Tensor] = None
    rnorms: Optional[torch.Tensor] = None

    @property
    def shape(self):
        return tuple(self.norms.shape)

    def view(self) -> L.TqCacheView:
        # built once per (arrays, layout): a decode step passes the same views
        key = (_ptr(self.codes), _ptr(self.qjl), _ptr(self.norms), _ptr(self.rnorms), self.norms.stride())
        cached = self.__dict__.get("_view")
        if cached is not None and cached[0] == key:
            return cached[1]
        sb, sh, sn = key[4]
        for t in (self.codes, self.qjl, self.rnorms):
            if t is not None:
                w = t.shape[3] if t.dim() == 4 else 1
                assert t.stride()[:3] == (sb * w, sh * w, sn * w), "all arrays must share one record layout"
        v = L.TqCacheView(key[0], key[1], key[2], key[3], sb, sh, sn)
        self.__dict__["_view"] = (key, v)
        return v

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.qjl, self.norms, self.rnorms)
                   if t is not None)


def empty_cache(qz: Quantizer, B: int, H: int, N: int, device="cuda") -> PackedCache:
    dev = torch.device(device)
    codes = torch.empty((B, H, N, qz.code_bytes), dtype=torch.uint8, device=dev) if qz.bm > 0 else None
    qjl = torch.empty((B, H, N, qz.qjl_bytes), dtype=torch.uint8, device=dev) if qz.prod else None
    rn = torch.empty((B, H, N), dtype=torch.float32, device=dev) if qz.prod else None
    return PackedCache(codes, torch.empty((B, H, N), dtype=torch.float32, device=dev), qjl, rn)


def _as_bhn(x: torch.Tensor) -> torch.Tensor:
    if x.dim() == 2:
        return x[None, None]
    if x.dim() == 3:
        return x[None]
    return x


# ------------------------------------------------------------- device calls

def encode(qz: Quantizer, x: torch.Tensor, out: Optional[PackedCache] = None, stream=None) -> PackedCache:
    """tq_encode of x shaped [B, H, N, d] (or [H, N, d] / [N, d]); the last
    dim must be contiguous; out defaults to a new [B, H, N] cache."""
    x4 = _as_bhn(x)
    B, H, N, d = x4.shape
    # a channel-group quantizer reads its channels of a wider row
    assert (d == qz.d if qz.channels is None else d >= qz.d) and x4.stride(3) == 1 and x4.dtype in _DTYPES
    if out is None:
        out = empty_cache(qz, B, H, N, x.device)
    v = out.view()
    L.check(L.lib().tq_encode(ctypes.byref(qz.c_struct()), x4.data_ptr(), _DTYPES[x4.dtype], B, H, N,
                              x4.stride(0), x4.stride(1), x4.stride(2), ctypes.byref(v), _stream(stream)))
    return out


def dequant(qz: Quantizer, cache: PackedCache, stream=None) -> torch.Tensor:
    """tq_dequant into a new fp32 tensor [B, H, N, d]."""
    B, H, N = cache.shape
    out = torch.empty((B, H, N, qz.d), dtype=torch.float32, device=cache.norms.device)
    v = cache.view()
    L.check(L.lib().tq_dequant(ctypes.byref(qz.c_struct()), ctypes.byref(v), B, H, N, out.data_ptr(),
                               _stream(stream)))
    return out


def decode_workspace_bytes(B: int, Hq: int, Hkv: int, seq_len: int, d: int) -> int:
    return int(L.lib().tq_decode_workspace_bytes(B, Hq, Hkv, seq_len, d))


class DecodeAttention:
    """Reusable tq_decode_attention call with its workspace allocated once
    (so that repeated steps allocate nothing)."""

    def __init__(self, kq: Quantizer, vq: Quantizer, B: int, Hq: int, Hkv: int, seq_len: int,
                 device="cuda"):
        self.kq, self.vq = kq, vq
        self.B, self.Hq, self.Hkv, self.seq_len = B, Hq, Hkv, seq_len
        nb = decode_workspace_bytes(B, Hq, Hkv, seq_len, kq.d)
        self.workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)
        self.ws_bytes = nb
        self.out = torch.empty((B, Hq, kq.d), dtype=torch.float32, device=device)

    def __call__(self, q: torch.Tensor, kcache: PackedCache, vcache: PackedCache, scale: Optional[float] = None,
                 seq_lens: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        B, Hq, d = q.shape
        assert (B, Hq) == (self.B, self.Hq) and q.is_contiguous() and q.dtype in _DTYPES
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        out = self.out if out is None else out
        kv, vv = kcache.view(), vcache.view()
        if seq_lens is not None:
            assert seq_lens.dtype == torch.int32 and seq_lens.is_contiguous()
        L.check(L.lib().tq_decode_attention(
            ctypes.byref(self.kq.c_struct()), ctypes.byref(self.vq.c_struct()), q.data_ptr(), _DTYPES[q.dtype],
            B, Hq, self.Hkv, self.seq_len, _ptr(seq_lens), ctypes.byref(kv), ctypes.byref(vv), float(scale),
            out.data_ptr(), _ptr(scores), self.workspace.data_ptr(), self.ws_bytes, _stream(stream)))
        return out

    def append_step(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_tail: PackedCache,
                    v_tail: PackedCache, kcache: PackedCache, vcache: PackedCache, scale: Optional[float] = None,
                    seq_lens: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """tq_append_decode_attention: encode the new token's K and V
        ([B, Hkv, d] or [B, Hkv, 1, d], same dtype) into the tail records
        k_tail / v_tail ([B, Hkv, 1] views, usually the last token of
        kcache / vcache), then attend over kcache / vcache."""
        B, Hq, d = q.shape
        assert (B, Hq) == (self.B, self.Hq) and q.is_contiguous() and q.dtype in _DTYPES
        if k_new.dim() == 4:
            k_new, v_new = k_new[:, :, 0], v_new[:, :, 0]
        assert k_new.shape == (B, self.Hkv, d) and v_new.shape == k_new.shape
        assert k_new.dtype == v_new.dtype and k_new.dtype in _DTYPES
        assert k_new.stride() == v_new.stride() and k_new.stride(2) == 1
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        out = self.out if out is None else out
        kv, vv, kt, vt = kcache.view(), vcache.view(), k_tail.view(), v_tail.view()
        if seq_lens is not None:
            assert seq_lens.dtype == torch.int32 and seq_lens.is_contiguous()
        L.check(L.lib().tq_append_decode_attention(
            ctypes.byref(self.kq.c_struct()), ctypes.byref(self.vq.c_struct()), k_new.data_ptr(), v_new.data_ptr(),
            _DTYPES[k_new.dtype], k_new.stride(0), k_new.stride(1), ctypes.byref(kt), ctypes.byref(vt),
            q.data_ptr(), _DTYPES[q.dtype], B, Hq, self.Hkv, self.seq_len, _ptr(seq_lens), ctypes.byref(kv),
            ctypes.byref(vv), float(scale), out.data_ptr(), _ptr(scores), self.workspace.data_ptr(), self.ws_bytes,
            _stream(stream)))
        return out


def decode_attention(kq: Quantizer, vq: Quantizer, q: torch.Tensor, kcache: PackedCache, vcache: PackedCache,
                     scale: Optional[float] = None, seq_lens: Optional[torch.Tensor] = None,
                     scores: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One-shot tq_decode_attention (allocates its workspace and output)."""
    B, Hq, _ = q.shape
    _, Hkv, N = kcache.shape
    op = DecodeAttention(kq, vq, B, Hq, Hkv, N, device=q.device)
    return op(q, kcache, vcache, scale=scale, seq_lens=seq_lens, scores=scores).clone()


class SplitQuantizer:
    """Outlier-channel split of a d-channel head: group 0 (the outlier
    channels, ascending) at bits_o, group 1 (the rest) at bits_r, each its
    own dense-rotation quantizer reading its channels of the head."""

    def __init__(self, d: int, channels, bits_o: int, bits_r: int, variant: str = "mse", seed_rot: int = 0,
                 seed_qjl: int = 1, device="cuda"):
        ch = torch.as_tensor(channels, dtype=torch.int64).sort().values
        mask = torch.ones(d, dtype=torch.bool)
        mask[ch] = False
        rest = torch.nonzero(mask)[:, 0]
        self.d, self.channels, self.rest = d, ch, rest
        self.groups = (
            Quantizer(ch.numel(), bits_o, variant, seed_rot=seed_rot, seed_qjl=seed_qjl, device=device,
                      rotation="dense", channels=ch),
            Quantizer(rest.numel(), bits_r, variant, seed_rot=seed_rot + 1, seed_qjl=seed_qjl + 1, device=device,
                      rotation="dense", channels=rest))

    def c_array(self):
        return (L.TqQuantizer * 2)(self.groups[0].c_struct(), self.groups[1].c_struct())


def encode_split(sq: SplitQuantizer, x: torch.Tensor, stream=None):
    """tq_encode of both channel groups of x ([B, H, N, d] or fewer dims):
    (cache of group 0, cache of group 1)."""
    return tuple(encode(g, x, stream=stream) for g in sq.groups)


class DecodeAttentionSplit:
    """tq_decode_attention_split with its workspace allocated once."""

    def __init__(self, kq: SplitQuantizer, vq: SplitQuantizer, B: int, Hq: int, Hkv: int, seq_len: int,
                 device="cuda"):
        self.kq, self.vq, self.B, self.Hq, self.Hkv, self.seq_len = kq, vq, B, Hq, Hkv, seq_len
        nb = int(L.lib().tq_decode_split_workspace_bytes(B, Hq, Hkv, seq_len, kq.d))
        self.workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)
        self.ws_bytes = nb
        self.out = torch.empty((B, Hq, kq.d), dtype=torch.float32, device=device)

    def __call__(self, q: torch.Tensor, kcaches, vcaches, scale: Optional[float] = None,
                 seq_lens: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        B, Hq, d = q.shape
        assert (B, Hq, d) == (self.B, self.Hq, self.kq.d) and q.is_contiguous() and q.dtype in _DTYPES
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        kv = (L.TqCacheView * 2)(kcaches[0].view(), kcaches[1].view())
        vv = (L.TqCacheView * 2)(vcaches[0].view(), vcaches[1].view())
        ka, va = self.kq.c_array(), self.vq.c_array()
        L.check(L.lib().tq_decode_attention_split(
            ka, va, q.data_ptr(), _DTYPES[q.dtype], B, Hq, self.Hkv, self.seq_len, _ptr(seq_lens), kv, vv,
            float(scale), self.out.data_ptr(), self.workspace.data_ptr(), self.ws_bytes, _stream(stream)))
        return self.out


class Search:
    """Reusable tq_search_topk call over a packed database of n_db records
    (its workspace allocated once)."""

    def __init__(self, qz: Quantizer, n_q: int, n_db: int, device="cuda"):
        self.qz, self.n_q, self.n_db = qz, n_q, n_db
        nb = int(L.lib().tq_search_workspace_bytes(n_q, n_db, qz.d))
        self.workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)
        self.ws_bytes = nb

    def __call__(self, queries: torch.Tensor, db: PackedCache, k: int, stream=None):
        """(top scores [n_q, k] fp32, top indices [n_q, k] int64) of the
        queries [n_q, d] against the n_db records of db (shaped [1, 1, n_db]
        or [n_db], any record stride)."""
        n_q, d = queries.shape
        assert n_q == self.n_q and d == self.qz.d and queries.is_contiguous() and queries.dtype in _DTYPES
        dev = queries.device
        top_v = torch.empty((n_q, k), dtype=torch.float32, device=dev)
        top_i = torch.empty((n_q, k), dtype=torch.int64, device=dev)
        v = db.view()
        L.check(L.lib().tq_search_topk(ctypes.byref(self.qz.c_struct()), ctypes.byref(v), self.n_db,
                                       queries.data_ptr(), _DTYPES[queries.dtype], n_q, k, top_v.data_ptr(),
                                       top_i.data_ptr(), self.workspace.data_ptr(), self.ws_bytes,
                                       _stream(stream)))
        return top_v, top_i


def search_topk(qz: Quantizer, queries: torch.Tensor, db: PackedCache, k: int):
    """One-shot tq_search_topk (allocates its workspace and outputs)."""
    n_db = db.norms.numel()
    return Search(qz, queries.shape[0], n_db, device=queries.device)(queries, db, k)


def set_decode_feed(staged: bool) -> bool:
    """Feed of the tensor-core decode for this process: bulk-copy staging
    through shared memory (True) or straight into registers (False, the
    default). Returns whether staging was on before."""
    prev = L.lib().tq_set_decode_feed(L.TQ_FEED_BULK_STAGED if staged else L.TQ_FEED_REGISTERS)
    return prev == L.TQ_FEED_BULK_STAGED


def check(stream=None) -> None:
    L.check(L.lib().tq_check(_stream(stream)))
