"""ctypes view of libkvdecode.so (include/kvdecode.h).

Loading fails loudly: there is no fallback implementation of any entry point.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvdecode.so")

KVD_OK = 0
KVD_ERR_INVALID_ARG = -1
KVD_ERR_UNSUPPORTED = -2
KVD_ERR_WORKSPACE = -3
KVD_ERR_CUDA = -4

KVD_F32 = 0
KVD_BF16 = 1

KVD_FLAG_PAGE_OUT_OF_RANGE = 0x1
KVD_FLAG_CAPACITY = 0x2
KVD_FLAG_WAIT_TIMEOUT = 0x4

KVD_STATIC_WORKSPACE_BYTES = 16 << 20

# Every exported symbol of include/kvdecode.h with its ctypes signature.
c_int, c_size_t, c_void_p, c_char_p = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_char_p


class Params(ctypes.Structure):
    """Mirror of ``kvd_params``."""
    _fields_ = [
        ("batch", c_int),
        ("num_heads", c_int),
        ("num_kv_heads", c_int),
        ("head_dim", c_int),
        ("q_len", c_int),
        ("scale", ctypes.c_float),
        ("rope_base", ctypes.c_float),
        ("dtype", c_int),
        ("out_dtype", c_int),
        ("max_seq_len", c_int),
        ("page_size", c_int),
        ("num_pages", c_int),
        ("max_pages_per_seq", c_int),
        ("max_kv_len", c_int),
        ("status", c_void_p),
        ("rope_interleaved", c_int),
        ("rotary_dim", c_int),
    ]


PP = ctypes.POINTER(Params)

SIGNATURES = {
    "kv_append_rope": (c_int, [PP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_void_p]),
    "decode_attention": (c_int, [PP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_size_t, c_void_p]),
    "decode_attention_paged": (c_int, [PP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_size_t, c_void_p]),
    "decode_attention_static": (c_int, [PP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_void_p]),
    "kvd_workspace_size": (c_size_t, [PP]),
    "kvd_decode_step": (c_int, [PP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "kv_append_rope_cow": (c_int, [PP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   c_void_p, c_void_p, c_void_p, c_void_p]),
    "kv_append_rope_shard": (c_int, [PP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_void_p]),
    "decode_attention_shard": (c_int, [PP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_size_t, c_void_p]),
    "kvd_merge_partials": (c_int, [PP, c_void_p, c_void_p, c_int, c_void_p, c_void_p]),
    "kvd_status_string": (c_char_p, [c_int]),
    "kvd_version": (c_int, []),
}

_LIB = None


class KvdError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = get_lib().kvd_status_string(status).decode()
        super().__init__(f"{fn} failed: {msg} (status {status})")
        self.status = status


def get_lib() -> ctypes.CDLL:
    """Load libkvdecode.so from the package directory (built in-tree)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m kv_cache_decode_rope_b200.build`; "
                "the decode path has no CPU fallback")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def check(fn: str, status: int) -> None:
    if status != KVD_OK:
        raise KvdError(fn, status)
