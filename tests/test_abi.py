"""The C-ABI library loads, exports every symbol the header declares, and its
host-side validation answers without a GPU (no kernel is launched by any call
here: each one fails a check before the first CUDA call)."""
import ctypes
import os
import re

import pytest

from kv_cache_decode_rope_b200 import _lib
from kv_cache_decode_rope_b200 import build as kvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_symbols():
    names = []
    for h in HEADERS:
        src = open(h).read()
        names += re.findall(r"KVD_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


@pytest.fixture(scope="module")
def lib():
    kvbuild.build()
    return _lib.get_lib()


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ("kv_append_rope", "decode_attention", "decode_attention_paged", "kvd_workspace_size",
              "kvd_status_string", "kvd_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_symbols():
        assert hasattr(lib, n), f"libkvdecode.so does not export {n}"
        assert n in _lib.SIGNATURES, f"binding lacks a signature for {n}"


def test_status_strings(lib):
    assert lib.kvd_status_string(0) == b"ok"
    for s in (-1, -2, -3, -4):
        assert lib.kvd_status_string(s) not in (b"ok", b"unknown status")
    assert lib.kvd_status_string(12345) == b"unknown status"
    assert lib.kvd_version() >= 100


def params(**kw):
    d = dict(batch=2, num_heads=8, num_kv_heads=2, head_dim=128, q_len=1, scale=0.088,
             rope_base=10000.0, dtype=_lib.KVD_BF16, out_dtype=_lib.KVD_F32, max_seq_len=64,
             page_size=16, num_pages=8, max_pages_per_seq=4, max_kv_len=64)
    d.update(kw)
    p = _lib.Params()
    for k, v in d.items():
        setattr(p, k, v)
    return p


FAKE = 4096  # 16-byte aligned, never dereferenced: every call below fails validation first


def call_decode(lib, p, ws_bytes=None, q=FAKE, ws=FAKE, paged=False):
    need = lib.kvd_workspace_size(ctypes.byref(p))
    nb = need if ws_bytes is None else ws_bytes
    if paged:
        return lib.decode_attention_paged(ctypes.byref(p), q, FAKE, FAKE, FAKE, FAKE, FAKE, ws, nb, None)
    return lib.decode_attention(ctypes.byref(p), q, FAKE, FAKE, FAKE, FAKE, ws, nb, None)


def test_null_params(lib):
    assert lib.decode_attention(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert lib.kv_append_rope(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == -1
    assert lib.kvd_workspace_size(None) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(num_heads=6, num_kv_heads=4), -1),        # Hq % Hkv != 0
    (dict(num_kv_heads=0), -1),
    (dict(head_dim=96), -2),                         # no kernel for D = 96
    (dict(head_dim=256, dtype=_lib.KVD_F32), -2),    # fp32 rows of 1 KB do not fit one warp
    (dict(dtype=7), -1),
    (dict(out_dtype=3), -1),
    (dict(num_heads=256, num_kv_heads=1), -2),      # 256 rows per unit > 128 (tensor-core path)
    (dict(num_heads=128, num_kv_heads=1, dtype=_lib.KVD_F32), -2),  # > 64 rows on the CUDA-core path
    (dict(num_heads=128, num_kv_heads=1, head_dim=64), -2),
    (dict(max_seq_len=0), -1),
    (dict(max_kv_len=0), -1),
    (dict(scale=float("nan")), -1),
])
def test_decode_validation(lib, kw, code):
    assert call_decode(lib, params(**kw)) == code


def test_decode_workspace_checks(lib):
    p = params()
    need = lib.kvd_workspace_size(ctypes.byref(p))
    assert need > 0 and need % 256 == 0
    assert call_decode(lib, p, ws_bytes=need - 1) == -3
    assert call_decode(lib, p, ws=0) == -3
    assert call_decode(lib, p, ws=FAKE + 8) == -3   # misaligned workspace


def test_decode_pointer_checks(lib):
    assert call_decode(lib, params(), q=0) == -1
    assert call_decode(lib, params(), q=FAKE + 2) == -1


@pytest.mark.parametrize("kw,code", [
    (dict(page_size=8), -2), (dict(page_size=24), -2), (dict(num_pages=0), -1),
    (dict(max_pages_per_seq=0), -1)])
def test_paged_validation(lib, kw, code):
    assert call_decode(lib, params(**kw), paged=True) == code


def test_paged_requires_table(lib):
    p = params()
    need = lib.kvd_workspace_size(ctypes.byref(p))
    assert lib.decode_attention_paged(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE,
                                      need, None) == -1


def test_append_validation(lib):
    def app(p, q=FAKE):
        return lib.kv_append_rope(ctypes.byref(p), q, FAKE, FAKE, FAKE, FAKE, FAKE, None, None)
    assert app(params(rotary_dim=24)) == -2          # not a multiple of 16
    assert app(params(rotary_dim=256)) == -2         # wider than head_dim
    assert app(params(rotary_dim=8, head_dim=16)) == -2
    assert app(params(rope_interleaved=2)) == -1
    assert app(params(rope_base=0.0)) == -1
    assert app(params(rope_base=float("inf"))) == -1
    assert app(params(head_dim=48)) == -2
    assert app(params(), q=0) == -1
    assert app(params(), q=FAKE + 4) == -1


def test_empty_problems_are_noops(lib):
    # B = 0 or q_len = 0: nothing to do, success without touching the device
    assert call_decode(lib, params(batch=0), ws=0, ws_bytes=0) in (0, -3)
    p = params(q_len=0)
    assert lib.decode_attention(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None) == 0
    assert lib.kv_append_rope(ctypes.byref(params(batch=0)), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              None, None) == 0


def test_workspace_size_grows_with_problem(lib):
    small = lib.kvd_workspace_size(ctypes.byref(params(batch=1)))
    big = lib.kvd_workspace_size(ctypes.byref(params(batch=64)))
    rows = lib.kvd_workspace_size(ctypes.byref(params(q_len=4)))
    assert 0 < small < big
    assert rows > lib.kvd_workspace_size(ctypes.byref(params()))


def call_static(lib, p, q=FAKE, paged=False):
    return lib.decode_attention_static(ctypes.byref(p), q, FAKE, FAKE, FAKE, FAKE if paged else None,
                                       FAKE, None)


STATIC_CASES = [
    dict(num_heads=6, num_kv_heads=4), dict(num_kv_heads=0), dict(head_dim=96),
    dict(head_dim=256, dtype=_lib.KVD_F32), dict(dtype=7), dict(out_dtype=3),
    dict(num_heads=256, num_kv_heads=1), dict(num_heads=128, num_kv_heads=1, dtype=_lib.KVD_F32),
    dict(max_seq_len=0), dict(max_kv_len=0), dict(scale=float("nan")),
    # no work, but a configuration no kernel supports: refused all the same
    dict(batch=0, head_dim=48), dict(q_len=0, head_dim=96), dict(batch=0, dtype=7),
    dict(batch=0, max_seq_len=0),
]


@pytest.mark.parametrize("kw", STATIC_CASES)
def test_static_entry_validates_like_decode_attention(lib, kw):
    """decode_attention_static answers every rejected configuration exactly as
    decode_attention does, before any CUDA call (these run without a GPU)."""
    p = params(**kw)
    ref = lib.decode_attention(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert ref != 0
    assert call_static(lib, p) == ref


@pytest.mark.parametrize("kw", [dict(page_size=8), dict(num_pages=0), dict(max_pages_per_seq=0)])
def test_static_entry_paged_validation(lib, kw):
    p = params(**kw)
    assert call_static(lib, p, paged=True) == call_decode(lib, p, paged=True) != 0


def test_static_entry_pointer_checks_and_empty_calls(lib):
    assert lib.decode_attention_static(None, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == -1
    assert call_static(lib, params(), q=0) == -1
    assert call_static(lib, params(), q=FAKE + 2) == -1
    assert call_static(lib, params(batch=0)) == 0
    assert call_static(lib, params(q_len=0), paged=True) == 0
