"""The C-ABI library loads, exports every symbol include/slc.h declares, and
rejects bad arguments before touching the GPU.  CPU only: no compute call
is made (validation errors return before any CUDA call)."""
import ctypes
import os
import re
import subprocess

import pytest

import sparse_long_context_max_b200 as slc
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "slc.h")
lib = slc._lib

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, -1, -2, -3


def declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SLC_API\s+[\w\s\*]+?\b(slc_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared()
    for want in ["slc_kv_append", "slc_build_page_meta", "slc_sparse_decode",
                 "slc_dense_decode", "slc_workspace_size", "slc_score_pages",
                 "slc_select_pages", "slc_select_pages_delta", "slc_sparse_decode_delta",
                 "slc_device_status", "slc_error_string"]:
        assert want in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", slc.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (slc_\w+)", out))
    missing = [n for n in declared() if n not in exported]
    assert not missing, missing
    for n in declared():
        assert hasattr(lib, n)


def test_error_strings():
    for code in (0, -1, -2, -3, -4, -5):
        assert lib.slc_error_string(code)
    assert lib.slc_error_string(-99) == b"unknown error"


def test_workspace_size():
    n = lib.slc_workspace_size(4, 32, 4, 128, 16400, 256)
    assert n > 4 * 4 * 16400 * 4  # at least the scores
    assert n % 256 == 0
    assert lib.slc_workspace_size(4, 32, 4, 128, 16400, 512) > n
    assert lib.slc_workspace_size(4, 32, 4, 64, 16400, 256) == 0  # head_dim
    assert lib.slc_workspace_size(4, 30, 4, 128, 16400, 256) == 0  # Hq % Hkv
    assert lib.slc_workspace_size(4, 36, 4, 128, 16400, 256) == 0  # group 9
    assert lib.slc_workspace_size(4, 32, 4, 128, 0, 256) == 0
    assert lib.slc_workspace_size(4, 32, 4, 128, 100, -1) == 0


FAKE = 0x10000  # a 16-byte aligned address that is never dereferenced


def cache(**kw):
    c = dict(k_cache=FAKE, v_cache=FAKE, meta=FAKE, num_pages=10, num_kv_heads=2,
             head_dim=128, page_size=16, meta_format=0)
    c.update(kw)
    return slc._Cache(**c)


def sparse(c, q=FAKE, hq=8, batch=1, max_pages=10, prefix=0, window=0, budget=2,
           scale=0.0, out=FAKE, ws=FAKE, ws_bytes=1 << 40):
    return lib.slc_sparse_decode(q, ctypes.byref(c), FAKE, max_pages, FAKE, batch, hq,
                                 prefix, window, budget, scale, out, None, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(page_size=32), UNSUPPORTED),
    (dict(head_dim=64), UNSUPPORTED),
    (dict(num_kv_heads=0), INVALID),
    (dict(num_pages=0), INVALID),
    (dict(k_cache=None), INVALID),
    (dict(meta=FAKE + 8), INVALID),  # misaligned
    (dict(meta_format=2), UNSUPPORTED),  # no such metadata format
])
def test_cache_validation(kw, code):
    assert sparse(cache(**kw)) == code


def test_decode_argument_validation():
    c = cache()
    assert sparse(c, hq=7) == INVALID  # Hq % Hkv
    assert sparse(c, hq=18) == UNSUPPORTED  # group 9 > 8
    assert sparse(c, budget=-1) == INVALID
    assert sparse(c, prefix=-1) == INVALID
    assert sparse(c, window=-5) == INVALID
    assert sparse(c, max_pages=0) == INVALID
    assert sparse(c, max_pages=40000) == UNSUPPORTED  # > 32768 candidates
    assert sparse(c, q=None) == INVALID
    assert sparse(c, q=FAKE + 2) == INVALID
    assert sparse(c, out=None) == INVALID
    assert sparse(c, ws=None) == INVALID
    assert sparse(c, scale=float("nan")) == INVALID
    assert sparse(c, ws_bytes=100) == WORKSPACE
    assert sparse(c, batch=0) == OK  # nothing to do, no CUDA call
    assert lib.slc_dense_decode(FAKE, ctypes.byref(c), FAKE, 10, FAKE, 1, 8, 0.0, FAKE, FAKE,
                                100, None) == WORKSPACE
    assert lib.slc_kv_append(ctypes.byref(c), None, FAKE, FAKE, 10, FAKE, 1, None) == INVALID
    assert lib.slc_kv_append(ctypes.byref(c), FAKE, FAKE, FAKE, 10, FAKE, 0, None) == OK
    assert lib.slc_build_page_meta(None, FAKE, 10, FAKE, 1, None) == INVALID
    assert lib.slc_select_pages(FAKE, 2, 10, FAKE, 1, 0, 0, -3, FAKE, None) == INVALID
    assert lib.slc_select_pages(FAKE, 2, 10, FAKE, 1, 0, 0, 0, FAKE, None) == OK
    assert lib.slc_score_pages(FAKE, ctypes.byref(c), FAKE, 10, FAKE, 1, 8, -1, 0, FAKE,
                               None) == INVALID
    # top-delta: d >= 0, cap >= 0, delta not NaN; nothing to do for cap 0 or batch 0
    sd = lib.slc_select_pages_delta
    assert sd(FAKE, 2, 10, FAKE, 1, 0, 0, -1, 1.0, 8, FAKE, None) == INVALID
    assert sd(FAKE, 2, 10, FAKE, 1, 0, 0, 4, float("nan"), 8, FAKE, None) == INVALID
    assert sd(FAKE, 2, 10, FAKE, 1, 0, 0, 4, 1.0, -1, FAKE, None) == INVALID
    assert sd(FAKE, 2, 40000, FAKE, 1, 0, 0, 4, 1.0, 8, FAKE, None) == UNSUPPORTED
    assert sd(FAKE, 2, 10, FAKE, 1, 0, 0, 4, float("inf"), 0, FAKE, None) == OK
    assert sd(FAKE, 2, 10, FAKE, 0, 0, 0, 4, 1.0, 8, FAKE, None) == OK
    dd = lib.slc_sparse_decode_delta
    assert dd(FAKE, ctypes.byref(c), FAKE, 10, FAKE, 1, 8, 0, 0, -2, 1.0, 4, 0.0, FAKE, None,
              FAKE, 1 << 40, None) == INVALID
    assert dd(FAKE, ctypes.byref(c), FAKE, 10, FAKE, 1, 8, 0, 0, 2, float("nan"), 4, 0.0, FAKE,
              None, FAKE, 1 << 40, None) == INVALID
    assert dd(FAKE, ctypes.byref(c), FAKE, 10, FAKE, 1, 8, 0, 0, 2, 1.0, -4, 0.0, FAKE, None,
              FAKE, 1 << 40, None) == INVALID
    assert dd(FAKE, ctypes.byref(c), FAKE, 10, FAKE, 1, 8, 0, 0, 2, 1.0, 4, 0.0, FAKE, None,
              FAKE, 100, None) == WORKSPACE
    assert lib.slc_device_status(None, None) == INVALID
    for stage in (0, 3, -1):  # only stages 1 and 2 exist
        assert lib.slc_sparse_decode_stage(stage, FAKE, ctypes.byref(c), FAKE, 10, FAKE, 1, 8, 0,
                                           0, 2, 0.0, FAKE, None, FAKE, 1 << 40,
                                           None) == INVALID
    assert lib.slc_sparse_decode_stage(2, FAKE, ctypes.byref(c), FAKE, 10, FAKE, 1, 7, 0, 0, 2,
                                       0.0, FAKE, None, FAKE, 1 << 40, None) == INVALID  # Hq % Hkv


def test_static_entry_checks_arguments_before_size():
    """The allocation-free entry runs the same argument checks as
    slc_sparse_decode, before its scratch-size test."""
    f = lib.slc_sparse_decode_static
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_void_p, ctypes.POINTER(slc._Cache), ctypes.c_void_p, ctypes.c_int32,
                  ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    c = cache()

    def call(batch=1, max_pages=10, prefix=0, window=0, budget=2, scale=0.0, q=FAKE, hq=8):
        return f(q, ctypes.byref(c), FAKE, max_pages, FAKE, batch, hq, prefix, window, budget,
                 scale, FAKE, None, None)
    # shapes whose workspace would not fit the scratch array, with a bad
    # argument: the argument error wins
    big = dict(batch=64, max_pages=32768, budget=4096)
    assert call(**big, prefix=-1) == INVALID
    assert call(**big, window=-1) == INVALID
    assert call(**big, scale=float("inf")) == INVALID
    assert call(64, 40000, budget=4096) == UNSUPPORTED  # > 32768 candidates
    assert call(**big, q=FAKE + 4) == INVALID
    assert call(**big) == WORKSPACE  # well-formed but too large
    assert call(batch=0) == OK


def test_binding_rejects_cpu_tensors():
    import torch
    k = torch.zeros((4, 2, 16, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        slc.PagedCache(k, k)
