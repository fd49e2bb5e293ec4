"""The C-ABI library on the CPU: it loads, exports what include/tq.h
declares, its host routines equal the oracle bit for bit, and argument
checks return the documented status before any launch (no GPU needed)."""

import ctypes
import os
import re

import numpy as np
import pytest

from kv_cache_vector_13_b200 import _lib as L
from kv_cache_vector_13_b200 import api
from oracle import codebook as cb
from oracle import prng

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = L.lib()
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.EXPORTS)
    assert lib.tq_version().startswith(b"tq-b200")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_codebook_bit_exact_with_oracle(d, b):
    c, t = api.make_codebook(d, b)
    c2, t2, _, _ = cb.codebook(d, b)
    np.testing.assert_array_equal(c, c2)
    np.testing.assert_array_equal(t, t2)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_beta_codebook_bit_exact_with_oracle(b):
    c, t = api.make_codebook(128, b, "beta")
    c2, t2, _, _ = cb.codebook(128, b, "beta")
    np.testing.assert_array_equal(c, c2)
    np.testing.assert_array_equal(t, t2)


@pytest.mark.parametrize("d", [8, 64, 128, 200, 256])
def test_dense_rotation_matches_oracle_within_one_ulp(d):
    # the library's Householder QR and the oracle's LAPACK QR, both in double
    # with the same sign fix, agree to within one fp32 rounding step
    from oracle import rotation as rot
    P = api.make_rotation(12345 + d, d)
    Q = rot.haar_matrix(12345 + d, d).astype(np.float32)
    ulp = np.abs(P.view(np.int32).astype(np.int64) - Q.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1
    assert (ulp > 0).mean() < 1e-3


@pytest.mark.parametrize("seed", [0, 1, 7, 2 ** 40 + 3, 2 ** 64 - 1])
def test_seeded_parameters_bit_exact_with_oracle(seed):
    np.testing.assert_array_equal(api.make_signs(seed, 256), prng.signs(seed, 256))
    np.testing.assert_array_equal(api.make_qjl(seed, 64), prng.gaussian_matrix(seed, 64))


def test_record_sizes():
    assert api.code_bytes(128, 4, "mse") == 64 and api.qjl_bytes(128, "mse") == 0
    assert api.code_bytes(128, 3, "prod") == 32 and api.qjl_bytes(128, "prod") == 16
    assert api.code_bytes(128, 1, "prod") == 0
    assert api.code_bytes(64, 3, "mse") == 24


# ------------------------------------------------------------------ validation

FAKE = 0x10000  # a 64 KiB-aligned address that is never dereferenced


def quant(d=128, bits=4, variant=L.TQ_MSE, rot=L.TQ_ROT_HADAMARD, ptrs=True, rot_matrix=None):
    p = FAKE if ptrs else None
    return L.TqQuantizer(d, bits, variant, rot, p, p, p, p, rot_matrix)


def view(codes=FAKE, norms=FAKE, qjl=FAKE, rnorms=FAKE, sb=0, sh=0, sn=1):
    return L.TqCacheView(codes, qjl, norms, rnorms, sb, sh, sn)


def enc(q, x=FAKE, dtype=L.TQ_F32, B=1, H=1, N=4, strides=(0, 0, 128), out=None):
    out = out if out is not None else view()
    return L.lib().tq_encode(ctypes.byref(q) if q is not None else None, x, dtype, B, H, N, *strides,
                             ctypes.byref(out), None)


def test_encode_argument_checks():
    assert enc(None) == L.TQ_EINVAL
    assert enc(quant(d=100)) == L.TQ_EINVAL
    assert enc(quant(bits=5)) == L.TQ_EINVAL
    assert enc(quant(bits=0)) == L.TQ_EINVAL
    assert enc(quant(variant=7)) == L.TQ_EINVAL
    assert enc(quant(rot=L.TQ_ROT_DENSE)) == L.TQ_EINVAL                        # no rot matrix
    assert enc(quant(rot=L.TQ_ROT_DENSE, rot_matrix=FAKE + 4)) == L.TQ_EINVAL   # misaligned
    assert enc(quant(d=100, rot=L.TQ_ROT_DENSE, rot_matrix=FAKE)) == L.TQ_EINVAL  # d not a multiple of 8
    assert enc(quant(d=200)) == L.TQ_EINVAL                                     # Hadamard needs 2^k
    assert enc(quant(ptrs=False)) == L.TQ_EINVAL
    assert enc(quant(), dtype=9) == L.TQ_EINVAL
    assert enc(quant(), B=-1) == L.TQ_EINVAL
    assert enc(quant(), x=FAKE + 4) == L.TQ_EINVAL            # x not 16-byte aligned
    assert enc(quant(), strides=(0, 0, 130)) == L.TQ_EINVAL    # stride * 4 not a multiple of 16
    assert enc(quant(), out=view(codes=FAKE + 8)) == L.TQ_EINVAL
    assert enc(quant(), out=view(norms=None)) == L.TQ_EINVAL
    assert enc(quant(variant=L.TQ_PROD), out=view(qjl=None)) == L.TQ_EINVAL
    assert enc(quant(), out=view(sn=-1)) == L.TQ_EINVAL
    assert "16-byte" in L.last_error() or "stride" in L.last_error()
    # empty work is a no-op that succeeds without touching any pointer
    assert enc(quant(), x=None, N=0) == L.TQ_OK


def dec(kq=None, vq=None, B=1, Hq=8, Hkv=2, N=100, ws_bytes=1 << 20, q=FAKE, out=FAKE, k=None, v=None,
        scale=0.1, ws=FAKE):
    kq = kq or quant()
    vq = vq or quant()
    k = k or view()
    v = v or view()
    return L.lib().tq_decode_attention(ctypes.byref(kq), ctypes.byref(vq), q, L.TQ_BF16, B, Hq, Hkv, N, None,
                                       ctypes.byref(k), ctypes.byref(v), scale, out, None, ws, ws_bytes, None)


def test_decode_argument_checks():
    need = L.lib().tq_decode_workspace_bytes(1, 8, 2, 100, 128)
    assert need > 0
    assert dec(Hq=6, Hkv=4) == L.TQ_EINVAL
    assert dec(Hkv=0) == L.TQ_EINVAL
    # prod values and d = 256 pass validation up to the workspace check (no
    # launch happens on these fake pointers)
    assert dec(vq=quant(variant=L.TQ_PROD), ws_bytes=need - 1) == L.TQ_EWORKSPACE
    need256 = L.lib().tq_decode_workspace_bytes(1, 8, 2, 100, 256)
    assert dec(kq=quant(d=256), vq=quant(d=256, variant=L.TQ_PROD), ws_bytes=need256 - 1) == L.TQ_EWORKSPACE
    assert dec(kq=quant(d=64), vq=quant(d=128)) == L.TQ_EINVAL
    assert dec(ws_bytes=need - 1) == L.TQ_EWORKSPACE
    assert dec(ws=FAKE + 4) == L.TQ_EWORKSPACE
    assert dec(q=FAKE + 2) == L.TQ_EINVAL
    assert dec(scale=float("nan")) == L.TQ_EINVAL
    assert dec(B=0) == L.TQ_OK


def test_workspace_query_edges():
    f = L.lib().tq_decode_workspace_bytes
    assert f(1, 8, 2, 0, 128) == 0
    assert f(1, 8, 3, 100, 128) == 0       # Hq not a multiple of Hkv
    assert f(1, 32, 8, 32768, 128) % 16 == 0
    assert f(1, 32, 8, 1 << 20, 128) >= f(1, 32, 8, 1 << 10, 128)


def test_noalloc_scratch_size_matches_header():
    # the binding's copy of TQ_NOALLOC_SCRATCH_BYTES is the header's value
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    m = re.search(r"#define\s+TQ_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", src)
    assert m, "TQ_NOALLOC_SCRATCH_BYTES not found in include/tq.h"
    assert L.TQ_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_status_strings():
    assert L.status_name(L.TQ_EWORKSPACE) == "TQ_EWORKSPACE"
    assert L.status_name(99) == "TQ_UNKNOWN"


def test_decode_feed_setter_round_trip():
    # the feed switch returns the previous setting and refuses unknown values
    lib = L.lib()
    prev = lib.tq_set_decode_feed(L.TQ_FEED_BULK_STAGED)
    try:
        assert prev in (L.TQ_FEED_REGISTERS, L.TQ_FEED_BULK_STAGED)
        assert lib.tq_set_decode_feed(7) == -1
        assert lib.tq_set_decode_feed(L.TQ_FEED_REGISTERS) == L.TQ_FEED_BULK_STAGED
        assert lib.tq_set_decode_feed(L.TQ_FEED_REGISTERS) == L.TQ_FEED_REGISTERS
    finally:
        lib.tq_set_decode_feed(prev if prev >= 0 else L.TQ_FEED_REGISTERS)
