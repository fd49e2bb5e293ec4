"""ctypes view of the C ABI declared in include/tq.h (libtq_b200.so).

Loading fails loudly when the library is missing: there is no fallback path.
"""

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_int64, c_size_t, c_uint64, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq_b200.so")

TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ECUDA, TQ_EWORKSPACE, TQ_ETIMEOUT = range(6)
TQ_FEED_REGISTERS, TQ_FEED_BULK_STAGED = 0, 1  # tq_decode_feed
TQ_MSE, TQ_PROD = 0, 1
TQ_ROT_HADAMARD, TQ_ROT_DENSE = 0, 1
TQ_CB_GAUSS, TQ_CB_BETA = 0, 1
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2
TQ_NOALLOC_SCRATCH_BYTES = 16 << 20  # include/tq.h

# every symbol include/tq.h declares
EXPORTS = (
    "tq_make_codebook", "tq_make_signs", "tq_make_qjl", "tq_make_rotation", "tq_code_bytes", "tq_qjl_bytes",
    "tq_encode", "tq_dequant", "tq_decode_workspace_bytes", "tq_decode_attention",
    "tq_append_decode_attention", "tq_decode_attention_noalloc",
    "tq_search_workspace_bytes", "tq_search_topk",
    "tq_decode_split_workspace_bytes", "tq_decode_attention_split",
    "tq_set_decode_feed", "tq_check", "tq_status_string", "tq_last_error", "tq_version",
)


class TqQuantizer(ctypes.Structure):
    _fields_ = [
        ("d", c_int32), ("bits", c_int32), ("variant", c_int32), ("rotation", c_int32),
        ("centroids", c_void_p), ("thresholds", c_void_p), ("signs", c_void_p), ("qjl_S", c_void_p),
        ("rot", c_void_p), ("channels", c_void_p),
    ]


class TqCacheView(ctypes.Structure):
    _fields_ = [
        ("codes", c_void_p), ("qjl", c_void_p), ("norms", c_void_p), ("rnorms", c_void_p),
        ("stride_b", c_int64), ("stride_h", c_int64), ("stride_n", c_int64),
    ]


class TqError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{status_name(status)}: {msg}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m kv_cache_vector_13_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    L.tq_make_codebook.argtypes = [c_int32, c_int32, c_int32, POINTER(c_float), POINTER(c_float)]
    L.tq_make_codebook.restype = c_int32
    L.tq_make_signs.argtypes = [c_uint64, c_int32, c_void_p]
    L.tq_make_signs.restype = c_int32
    L.tq_make_qjl.argtypes = [c_uint64, c_int32, POINTER(c_float)]
    L.tq_make_qjl.restype = c_int32
    L.tq_make_rotation.argtypes = [c_uint64, c_int32, POINTER(c_float)]
    L.tq_make_rotation.restype = c_int32
    L.tq_code_bytes.argtypes = [c_int32, c_int32, c_int32]
    L.tq_code_bytes.restype = c_size_t
    L.tq_qjl_bytes.argtypes = [c_int32, c_int32]
    L.tq_qjl_bytes.restype = c_size_t
    L.tq_encode.argtypes = [POINTER(TqQuantizer), c_void_p, c_int32, c_int64, c_int64, c_int64,
                            c_int64, c_int64, c_int64, POINTER(TqCacheView), c_void_p]
    L.tq_encode.restype = c_int32
    L.tq_dequant.argtypes = [POINTER(TqQuantizer), POINTER(TqCacheView), c_int64, c_int64, c_int64,
                             c_void_p, c_void_p]
    L.tq_dequant.restype = c_int32
    L.tq_decode_workspace_bytes.argtypes = [c_int32, c_int32, c_int32, c_int64, c_int32]
    L.tq_decode_workspace_bytes.restype = c_size_t
    L.tq_decode_attention.argtypes = [
        POINTER(TqQuantizer), POINTER(TqQuantizer), c_void_p, c_int32, c_int32, c_int32, c_int32,
        c_int64, c_void_p, POINTER(TqCacheView), POINTER(TqCacheView), c_float, c_void_p, c_void_p,
        c_void_p, c_size_t, c_void_p]
    L.tq_decode_attention.restype = c_int32
    L.tq_append_decode_attention.argtypes = [
        POINTER(TqQuantizer), POINTER(TqQuantizer), c_void_p, c_void_p, c_int32, c_int64, c_int64,
        POINTER(TqCacheView), POINTER(TqCacheView), c_void_p, c_int32, c_int32, c_int32, c_int32, c_int64,
        c_void_p, POINTER(TqCacheView), POINTER(TqCacheView), c_float, c_void_p, c_void_p, c_void_p, c_size_t,
        c_void_p]
    L.tq_append_decode_attention.restype = c_int32
    L.tq_decode_attention_noalloc.argtypes = [
        POINTER(TqQuantizer), POINTER(TqQuantizer), c_void_p, c_int32, c_int32, c_int32, c_int32,
        c_int64, c_void_p, POINTER(TqCacheView), POINTER(TqCacheView), c_float, c_void_p, c_void_p,
        c_void_p]
    L.tq_decode_attention_noalloc.restype = c_int32
    L.tq_search_workspace_bytes.argtypes = [c_int32, c_int64, c_int32]
    L.tq_search_workspace_bytes.restype = c_size_t
    L.tq_search_topk.argtypes = [POINTER(TqQuantizer), POINTER(TqCacheView), c_int64, c_void_p, c_int32, c_int32,
                                 c_int32, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]
    L.tq_search_topk.restype = c_int32
    L.tq_decode_split_workspace_bytes.argtypes = [c_int32, c_int32, c_int32, c_int64, c_int32]
    L.tq_decode_split_workspace_bytes.restype = c_size_t
    L.tq_decode_attention_split.argtypes = [
        POINTER(TqQuantizer), POINTER(TqQuantizer), c_void_p, c_int32, c_int32, c_int32, c_int32, c_int64,
        c_void_p, POINTER(TqCacheView), POINTER(TqCacheView), c_float, c_void_p, c_void_p, c_size_t, c_void_p]
    L.tq_decode_attention_split.restype = c_int32
    L.tq_set_decode_feed.argtypes = [c_int32]
    L.tq_set_decode_feed.restype = c_int32
    L.tq_check.argtypes = [c_void_p]
    L.tq_check.restype = c_int32
    L.tq_status_string.argtypes = [c_int32]
    L.tq_status_string.restype = c_char_p
    L.tq_last_error.argtypes = []
    L.tq_last_error.restype = c_char_p
    L.tq_version.argtypes = []
    L.tq_version.restype = c_char_p
    _lib = L
    return L


def status_name(s: int) -> str:
    return lib().tq_status_string(s).decode()


def last_error() -> str:
    return lib().tq_last_error().decode()


def check(status: int) -> None:
    if status != TQ_OK:
        raise TqError(status, last_error())
