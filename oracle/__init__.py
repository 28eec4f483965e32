"""CPU oracle for decode-step combined sparse attention (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  It is an independent, plain,
double-precision restatement of the method (see ``slc_oracle.c`` for the
steps and the readings taken) and shares no code with the CUDA library.

bf16 inputs are passed as their raw 16-bit patterns; torch bf16 tensors are
accepted and viewed as such.  All outputs are numpy float64 / int32 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "slc_oracle.c")
_LIB = os.path.join(_HERE, "libslc_oracle.so")
_lock = threading.Lock()
_lib = None

PAGE = 16


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math) into oracle/libslc_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load(path=None):
    global _lib
    with _lock:
        if _lib is None or path is not None:
            lib = ctypes.CDLL(path or build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_page_ranges.argtypes = [I, I, I, P, P, P]
            lib.oracle_page_ranges.restype = None
            lib.oracle_page_bounds.argtypes = [P, I, I, I, P, I, P, I, P, P]
            lib.oracle_page_bounds.restype = I
            lib.oracle_page_scores.argtypes = [P, I, I, I, P, P, I, P, I, I, I, P]
            lib.oracle_page_scores.restype = None
            lib.oracle_select_pages.argtypes = [P, I, I, P, I, I, I, I, P, P]
            lib.oracle_select_pages.restype = None
            lib.oracle_select_pages_delta.argtypes = [P, I, I, P, I, I, I, I,
                                                      ctypes.c_double, I, P, P]
            lib.oracle_select_pages_delta.restype = None
            lib.oracle_attend.argtypes = [P, P, P, I, I, I, I, P, I, P, I, I, I,
                                          P, I, I, ctypes.c_double, P]
            lib.oracle_attend.restype = I
            lib.oracle_sparse_decode.argtypes = [P, P, P, I, I, I, I, P, I, P, I,
                                                 I, I, I, ctypes.c_double, P, P, P]
            lib.oracle_sparse_decode.restype = I
            lib.oracle_fp8_value.argtypes = [I]
            lib.oracle_fp8_value.restype = ctypes.c_double
            lib.oracle_fp8_round.argtypes = [ctypes.c_double, I]
            lib.oracle_fp8_round.restype = I
            lib.oracle_page_bounds_fp8.argtypes = [P, I, I, I, P, I, P, I, P, P]
            lib.oracle_page_bounds_fp8.restype = I
            if path is not None:
                return lib
            _lib = lib
    return _lib


class use_library:
    """Context manager: route every call through another build of the
    oracle (used by the tests that plant mistakes in a copy of it)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        lib = _load(self.path)
        _lib = lib
        return lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _bits(x) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 numpy array of its bit patterns."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch  # local: only to reinterpret the tensor's bytes
        return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns (uint16) or a torch bf16 tensor")
    return a


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def page_ranges(L: int, prefix: int, window: int):
    """(n, np, ws): page count, prefix pages [0,np), window pages [ws,n)."""
    lib = _load()
    n, npre, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    lib.oracle_page_ranges(int(L), int(prefix), int(window), ctypes.byref(n),
                           ctypes.byref(npre), ctypes.byref(ws))
    return n.value, npre.value, ws.value


def page_bounds(k_cache, block_table, seq_lens):
    """Elementwise key min/max per logical page: two float64 arrays
    [B][Hkv][max_pages][D]; pages past the sequence are NaN."""
    lib = _load()
    k = _bits(k_cache)
    bt, sl = _i32(block_table), _i32(seq_lens)
    num_pages, hkv, page, dim = k.shape
    assert page == PAGE
    B, max_pages = bt.shape
    kmin = np.full((B, hkv, max_pages, dim), np.nan)
    kmax = np.full((B, hkv, max_pages, dim), np.nan)
    rc = lib.oracle_page_bounds(_ptr(k), num_pages, hkv, dim, _ptr(bt), max_pages,
                                _ptr(sl), B, _ptr(kmin), _ptr(kmax))
    if rc:
        raise ValueError("block table entry outside the page pool")
    return kmin, kmax


def fp8_value(code: int) -> float:
    """Value of an E4M3 code (NaN codes: +-the largest bf16, the
    out-of-range bound of their sign)."""
    return _load().oracle_fp8_value(int(code))


def fp8_round(x: float, up: bool) -> int:
    """Outward rounding to E4M3: up -> smallest value >= x, else largest
    value <= x (0x7F / 0xFF beyond the range)."""
    return _load().oracle_fp8_round(float(x), int(bool(up)))


def fp8_decode(codes) -> np.ndarray:
    """E4M3 codes (any shape, uint8) -> float64 values."""
    table = np.array([fp8_value(c) for c in range(256)])
    return table[np.asarray(codes, dtype=np.uint8)]


def page_bounds_fp8(k_cache, block_table, seq_lens):
    """E4M3 page bounds, rounded outward: two uint8 code arrays
    [B][Hkv][max_pages][D] (kmin rounded down, kmax up); pages past the
    sequence are 0."""
    lib = _load()
    k = _bits(k_cache)
    bt, sl = _i32(block_table), _i32(seq_lens)
    num_pages, hkv, page, dim = k.shape
    B, max_pages = bt.shape
    kmin = np.zeros((B, hkv, max_pages, dim), dtype=np.uint8)
    kmax = np.zeros((B, hkv, max_pages, dim), dtype=np.uint8)
    rc = lib.oracle_page_bounds_fp8(_ptr(k), num_pages, hkv, dim, _ptr(bt), max_pages,
                                    _ptr(sl), B, _ptr(kmin), _ptr(kmax))
    if rc:
        raise ValueError("block table entry outside the page pool")
    return kmin, kmax


def page_scores(q, kmin, kmax, seq_lens, prefix: int, window: int):
    """Quest bound per candidate page, float64 [B][Hkv][max_pages] (NaN
    outside the candidate range)."""
    lib = _load()
    qb = _bits(q)
    B, hq, dim = qb.shape
    kmin = np.ascontiguousarray(kmin, dtype=np.float64)
    kmax = np.ascontiguousarray(kmax, dtype=np.float64)
    _, hkv, max_pages, _ = kmin.shape
    sl = _i32(seq_lens)
    scores = np.empty((B, hkv, max_pages))
    lib.oracle_page_scores(_ptr(qb), hq, hkv, dim, _ptr(kmin), _ptr(kmax), max_pages,
                           _ptr(sl), B, int(prefix), int(window), _ptr(scores))
    return scores


def select_pages(scores, seq_lens, prefix: int, window: int, budget: int):
    """Top-budget candidate pages per (b, kv head): (sel [B][Hkv][budget]
    ascending, -1 padded; nsel [B][Hkv])."""
    lib = _load()
    s = np.ascontiguousarray(scores, dtype=np.float64)
    B, hkv, max_pages = s.shape
    sl = _i32(seq_lens)
    sel = np.empty((B, hkv, max(budget, 0)), dtype=np.int32)
    nsel = np.empty((B, hkv), dtype=np.int32)
    lib.oracle_select_pages(_ptr(s), hkv, max_pages, _ptr(sl), B, int(prefix),
                            int(window), int(budget), _ptr(sel), _ptr(nsel))
    return sel, nsel


def select_pages_delta(scores, seq_lens, prefix: int, window: int, d: int, delta: float,
                       cap: int):
    """Top-delta selection per (b, kv head): the d best candidates plus every
    candidate within delta of the best, ascending, -1 padded to cap (the cap
    best of the union if it is larger): (sel [B][Hkv][cap], nsel [B][Hkv])."""
    lib = _load()
    s = np.ascontiguousarray(scores, dtype=np.float64)
    B, hkv, max_pages = s.shape
    sl = _i32(seq_lens)
    sel = np.empty((B, hkv, max(cap, 1)), dtype=np.int32)
    nsel = np.empty((B, hkv), dtype=np.int32)
    lib.oracle_select_pages_delta(_ptr(s), hkv, max_pages, _ptr(sl), B, int(prefix),
                                  int(window), int(d), float(delta), int(cap), _ptr(sel),
                                  _ptr(nsel))
    return sel[:, :, :cap], nsel


def attend(q, k_cache, v_cache, block_table, seq_lens, prefix: int = 0,
           window: int = 0, sel=None, dense: bool = False, scale: float = 0.0):
    """Softmax attention over prefix + window + ``sel`` pages (or all pages
    when ``dense``).  Returns float64 [B][Hq][D]."""
    lib = _load()
    qb, k, v = _bits(q), _bits(k_cache), _bits(v_cache)
    bt, sl = _i32(block_table), _i32(seq_lens)
    B, hq, dim = qb.shape
    num_pages, hkv, _, _ = k.shape
    max_pages = bt.shape[1]
    if sel is None:
        sel = np.full((B, hkv, 0), -1, dtype=np.int32)
    sel = _i32(sel)
    budget = sel.shape[2]
    if budget == 0:
        sel = np.full((B, hkv, 1), -1, dtype=np.int32)
    out = np.zeros((B, hq, dim))
    rc = lib.oracle_attend(_ptr(qb), _ptr(k), _ptr(v), num_pages, hq, hkv, dim,
                           _ptr(bt), max_pages, _ptr(sl), B, int(prefix), int(window),
                           _ptr(sel), sel.shape[2], int(bool(dense)), float(scale),
                           _ptr(out))
    if rc:
        raise ValueError("block table entry outside the page pool")
    return out


def dense_decode(q, k_cache, v_cache, block_table, seq_lens, scale: float = 0.0):
    """Full attention over every token of every sequence."""
    return attend(q, k_cache, v_cache, block_table, seq_lens, dense=True, scale=scale)


def sparse_decode(q, k_cache, v_cache, block_table, seq_lens, prefix: int,
                  window: int, budget: int, scale: float = 0.0):
    """The whole decode step.  Returns (out [B][Hq][D] float64,
    sel [B][Hkv][budget] int32, nsel [B][Hkv] int32)."""
    lib = _load()
    qb, k, v = _bits(q), _bits(k_cache), _bits(v_cache)
    bt, sl = _i32(block_table), _i32(seq_lens)
    B, hq, dim = qb.shape
    num_pages, hkv, _, _ = k.shape
    max_pages = bt.shape[1]
    out = np.zeros((B, hq, dim))
    sel = np.empty((B, hkv, max(budget, 1)), dtype=np.int32)
    nsel = np.empty((B, hkv), dtype=np.int32)
    rc = lib.oracle_sparse_decode(_ptr(qb), _ptr(k), _ptr(v), num_pages, hq, hkv, dim,
                                  _ptr(bt), max_pages, _ptr(sl), B, int(prefix),
                                  int(window), int(budget), float(scale), _ptr(out),
                                  _ptr(sel), _ptr(nsel))
    if rc:
        raise ValueError("block table entry outside the page pool")
    return out, sel[:, :, :budget], nsel
