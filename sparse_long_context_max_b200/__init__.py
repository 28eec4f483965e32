"""Decode-step combined sparse attention on B200 (sm_100a).

A thin ctypes binding over the C ABI of ``libslc.so`` (include/slc.h): it
marshals torch CUDA tensors into pointers, sizes and the current CUDA stream.
Every step of the path runs in the library's kernels; there is no fallback.
Importing raises if the library cannot be loaded.

Tensors (all on the same CUDA device, contiguous):
    q            bf16  [B][Hq][D]
    k/v cache    bf16  [num_pages][Hkv][16][D]
    meta         bf16  [num_pages][Hkv][2][D]
    block_table  int32 [B][max_pages]
    seq_lens     int32 [B]
    out          fp32  [B][Hq][D]
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import _build

__all__ = [
    "SLCError", "PagedCache", "kv_append", "build_page_meta", "workspace_size",
    "score_pages", "select_pages", "select_pages_delta", "sparse_decode", "sparse_decode_delta",
    "sparse_attend", "dense_decode",
    "device_status",
    "library_path", "KERNELS_PER_CALL", "STATUS_BITS", "META_FORMATS",
]

PAGE = 16

# kernels one call launches (sparse decode and sparse attend: the streaming
# kernel, then the finishing kernel; dense: attend, merge)
KERNELS_PER_CALL = {"sparse_decode": 2, "sparse_decode_stage": 1, "dense_decode": 2,
                    "sparse_attend": 2, "kv_append": 1,
                    "build_page_meta": 1, "score_pages": 1, "select_pages": 1,
                    "select_pages_delta": 1, "sparse_decode_delta": 2}

STATUS_BITS = {1: "bad page", 2: "bad length", 4: "bad selection", 8: "wait timeout"}


class SLCError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(what)


class _Cache(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("meta", ctypes.c_void_p), ("num_pages", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("meta_format", ctypes.c_int32)]


# page metadata formats (include/slc.h SLC_META_*)
META_FORMATS = {"bf16": 0, "fp8": 1}


def _load() -> ctypes.CDLL:
    path = _build.LIB
    if _build.stale():
        path = _build.build()
    lib = ctypes.CDLL(path)
    P, I, Z, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    C = ctypes.POINTER(_Cache)
    sig = {
        "slc_kv_append": (I, [C, P, P, P, I, P, I, P]),
        "slc_build_page_meta": (I, [C, P, I, P, I, P]),
        "slc_workspace_size": (Z, [I, I, I, I, I, I]),
        "slc_score_pages": (I, [P, C, P, I, P, I, I, I, I, P, P]),
        "slc_select_pages": (I, [P, I, I, P, I, I, I, I, P, P]),
        "slc_select_pages_delta": (I, [P, I, I, P, I, I, I, I, F, I, P, P]),
        "slc_sparse_decode_delta": (I, [P, C, P, I, P, I, I, I, I, I, F, I, F, P, P, P, Z, P]),
        "slc_sparse_decode": (I, [P, C, P, I, P, I, I, I, I, I, F, P, P, P, Z, P]),
        "slc_dense_decode": (I, [P, C, P, I, P, I, I, F, P, P, Z, P]),
        "slc_sparse_attend": (I, [P, C, P, I, P, I, I, I, I, I, P, F, P, P, Z, P]),
        "slc_sparse_decode_stage": (I, [I, P, C, P, I, P, I, I, I, I, I, F, P, P, P, Z, P]),
        "slc_device_status": (I, [ctypes.POINTER(ctypes.c_int32), P]),
        "slc_error_string": (ctypes.c_char_p, [ctypes.c_int]),
        "slc_last_cuda_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def library_path() -> str:
    return _build.LIB


def _check(rc: int):
    if rc != 0:
        msg = _lib.slc_error_string(rc).decode()
        if rc == -4:
            msg += ": " + _lib.slc_last_cuda_error().decode()
        raise SLCError(rc, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims" % (name, ndim))
    return t


class PagedCache:
    """One layer's paged K/V cache plus its page metadata (device tensors).

    meta_format "bf16" keeps each page's key min/max exactly (bf16
    [num_pages][Hkv][2][D]); "fp8" keeps them as 8-bit E4M3 rounded outward
    (uint8, same shape: half the bytes the scoring reads)."""

    def __init__(self, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 meta: torch.Tensor | None = None, meta_format: str = "bf16"):
        _need(k_cache, torch.bfloat16, "k_cache", 4)
        _need(v_cache, torch.bfloat16, "v_cache", 4)
        if k_cache.shape != v_cache.shape or k_cache.shape[2] != PAGE:
            raise ValueError("k/v cache must be [num_pages][Hkv][16][D] and equal")
        if meta_format not in META_FORMATS:
            raise ValueError("meta_format must be one of %s" % sorted(META_FORMATS))
        n, hkv, _, d = k_cache.shape
        mdt = torch.bfloat16 if meta_format == "bf16" else torch.uint8
        if meta is None:
            meta = torch.empty((n, hkv, 2, d), dtype=mdt, device=k_cache.device)
        _need(meta, mdt, "meta", 4)
        if tuple(meta.shape) != (n, hkv, 2, d):
            raise ValueError("meta must be [num_pages][Hkv][2][D]")
        self.k_cache, self.v_cache, self.meta = k_cache, v_cache, meta
        self.meta_format = meta_format
        self.num_pages, self.num_kv_heads, self.head_dim = n, hkv, d
        self._c = _Cache(k_cache.data_ptr(), v_cache.data_ptr(), meta.data_ptr(), n, hkv, d, PAGE,
                         META_FORMATS[meta_format])

    @property
    def c(self):
        return ctypes.byref(self._c)


def kv_append(cache: PagedCache, k_new, v_new, block_table, positions):
    """Write one token per (sequence, kv head) and update its page bounds."""
    _need(k_new, torch.bfloat16, "k_new", 3)
    _need(v_new, torch.bfloat16, "v_new", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(positions, torch.int32, "positions", 1)
    B = positions.shape[0]
    _check(_lib.slc_kv_append(cache.c, _ptr(k_new), _ptr(v_new), _ptr(block_table),
                              block_table.shape[1], _ptr(positions), B, _stream()))


def build_page_meta(cache: PagedCache, block_table, seq_lens):
    """Rebuild every page's key min/max from the cache."""
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    _check(_lib.slc_build_page_meta(cache.c, _ptr(block_table), block_table.shape[1],
                                    _ptr(seq_lens), seq_lens.shape[0], _stream()))


def workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_pages, budget) -> int:
    n = _lib.slc_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_pages, budget)
    if n == 0 and batch > 0:
        raise SLCError(-2, "unsupported shape")
    return n


def score_pages(q, cache: PagedCache, block_table, seq_lens, prefix, window, scores=None):
    """fp32 [B][Hkv][max_pages] page scores (only candidate entries written)."""
    _need(q, torch.bfloat16, "q", 3)
    B, hq, _ = q.shape
    mp = block_table.shape[1]
    if scores is None:
        scores = torch.full((B, cache.num_kv_heads, mp), float("nan"), device=q.device)
    _need(scores, torch.float32, "scores", 3)
    _check(_lib.slc_score_pages(_ptr(q), cache.c, _ptr(block_table), mp, _ptr(seq_lens), B,
                                hq, prefix, window, _ptr(scores), _stream()))
    return scores


def select_pages(scores, seq_lens, prefix, window, budget, selected=None):
    """int32 [B][Hkv][budget] ascending selected pages, -1 padded."""
    _need(scores, torch.float32, "scores", 3)
    B, hkv, mp = scores.shape
    if selected is None:
        selected = torch.empty((B, hkv, budget), dtype=torch.int32, device=scores.device)
    _check(_lib.slc_select_pages(_ptr(scores), hkv, mp, _ptr(seq_lens), B, prefix, window,
                                 budget, _ptr(selected), _stream()))
    return selected


def select_pages_delta(scores, seq_lens, prefix, window, d, delta, cap, selected=None):
    """Top-delta selection: per (b, kv head) the d best candidate pages plus
    every candidate within delta of the best, at most cap; int32
    [B][Hkv][cap] ascending, -1 padded."""
    _need(scores, torch.float32, "scores", 3)
    B, hkv, mp = scores.shape
    if selected is None:
        selected = torch.empty((B, hkv, cap), dtype=torch.int32, device=scores.device)
    _check(_lib.slc_select_pages_delta(_ptr(scores), hkv, mp, _ptr(seq_lens), B, prefix, window,
                                       int(d), float(delta), int(cap), _ptr(selected),
                                       _stream()))
    return selected


_ws_cache: dict = {}


def _workspace(device, nbytes):
    buf = _ws_cache.get(device)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[device] = buf
    return buf


def sparse_decode(q, cache: PagedCache, block_table, seq_lens, prefix, window, budget,
                  scale=0.0, out=None, selected_out=None, workspace=None):
    """One sparse decode step of one layer; returns out (fp32 [B][Hq][D])."""
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    B, hq, d = q.shape
    mp = block_table.shape[1]
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out", 3)
    if selected_out is not None:
        _need(selected_out, torch.int32, "selected_out", 3)
    need = workspace_size(B, hq, cache.num_kv_heads, d, mp, budget)
    if workspace is None:
        workspace = _workspace(q.device, need)
    _check(_lib.slc_sparse_decode(_ptr(q), cache.c, _ptr(block_table), mp, _ptr(seq_lens), B,
                                  hq, prefix, window, budget, float(scale), _ptr(out),
                                  _ptr(selected_out), _ptr(workspace), workspace.numel(),
                                  _stream()))
    return out


def sparse_decode_delta(q, cache: PagedCache, block_table, seq_lens, prefix, window, d, delta,
                        cap, scale=0.0, out=None, selected_out=None, workspace=None):
    """One decode step with the top-delta selection (the d best candidate
    pages plus every candidate within delta of the best, at most cap) in
    place of the fixed budget; returns out (fp32 [B][Hq][D])."""
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    B, hq, dim = q.shape
    mp = block_table.shape[1]
    if out is None:
        out = torch.empty((B, hq, dim), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out", 3)
    if selected_out is not None:
        _need(selected_out, torch.int32, "selected_out", 3)
    need = workspace_size(B, hq, cache.num_kv_heads, dim, mp, cap)
    if workspace is None:
        workspace = _workspace(q.device, need)
    _check(_lib.slc_sparse_decode_delta(_ptr(q), cache.c, _ptr(block_table), mp, _ptr(seq_lens),
                                        B, hq, prefix, window, int(d), float(delta), int(cap),
                                        float(scale), _ptr(out), _ptr(selected_out),
                                        _ptr(workspace), workspace.numel(), _stream()))
    return out


def sparse_decode_stage(stage, q, cache: PagedCache, block_table, seq_lens, prefix, window,
                        budget, scale=0.0, out=None, selected_out=None, workspace=None):
    """One of the two kernels of sparse_decode alone: stage 1 the streaming
    kernel (prefix/window attention and candidate scores), stage 2 the
    finishing kernel (selection, selected-page attention, merge).  Stages 1
    then 2 on the same workspace equal one sparse_decode call."""
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    B, hq, d = q.shape
    mp = block_table.shape[1]
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out", 3)
    if selected_out is not None:
        _need(selected_out, torch.int32, "selected_out", 3)
    need = workspace_size(B, hq, cache.num_kv_heads, d, mp, budget)
    if workspace is None:
        workspace = _workspace(q.device, need)
    _check(_lib.slc_sparse_decode_stage(int(stage), _ptr(q), cache.c, _ptr(block_table), mp,
                                        _ptr(seq_lens), B, hq, prefix, window, budget,
                                        float(scale), _ptr(out), _ptr(selected_out),
                                        _ptr(workspace), workspace.numel(), _stream()))
    return out


def sparse_attend(q, cache: PagedCache, block_table, seq_lens, prefix, window, selected,
                  scale=0.0, out=None, workspace=None):
    """Attention over prefix, window and the given selection (int32
    [B][Hkv][budget], ascending, -1 padded; entries that are prefix or window
    pages add nothing); returns out (fp32 [B][Hq][D])."""
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    _need(selected, torch.int32, "selected", 3)
    B, hq, d = q.shape
    mp = block_table.shape[1]
    budget = selected.shape[2]
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out", 3)
    need = workspace_size(B, hq, cache.num_kv_heads, d, mp, budget)
    if workspace is None:
        workspace = _workspace(q.device, need)
    _check(_lib.slc_sparse_attend(_ptr(q), cache.c, _ptr(block_table), mp, _ptr(seq_lens), B,
                                  hq, prefix, window, budget, _ptr(selected), float(scale),
                                  _ptr(out), _ptr(workspace), workspace.numel(), _stream()))
    return out


def dense_decode(q, cache: PagedCache, block_table, seq_lens, scale=0.0, out=None,
                 workspace=None):
    """Full attention decode over every token; returns out (fp32 [B][Hq][D])."""
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    B, hq, d = q.shape
    mp = block_table.shape[1]
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out", 3)
    need = workspace_size(B, hq, cache.num_kv_heads, d, mp, 0)
    if workspace is None:
        workspace = _workspace(q.device, need)
    _check(_lib.slc_dense_decode(_ptr(q), cache.c, _ptr(block_table), mp, _ptr(seq_lens), B,
                                 hq, float(scale), _ptr(out), _ptr(workspace),
                                 workspace.numel(), _stream()))
    return out


def device_status() -> int:
    """Synchronise the current stream; return and clear the device status bits."""
    v = ctypes.c_int32(0)
    _check(_lib.slc_device_status(ctypes.byref(v), _stream()))
    return v.value
