"""The allocation-free decode entry point, through the C ABI.

Some callers cannot allocate device memory (for instance a plugin whose
host framework owns all GPU memory through its own pool), so they cannot
hand slc_sparse_decode a workspace.  slc_sparse_decode_static serves them
from a fixed scratch array inside the library.  These tests check that it
gives the same results as slc_sparse_decode (same tolerance as the other
GPU tests) on two calls in a row, and that it refuses shapes whose
workspace does not fit.  The file sorts last so that a run stopping at its
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from gpu_util import OUT_TOL

pytestmark = pytest.mark.gpu


def _lib():
    import sparse_long_context_max_b200 as slc
    lib = slc._lib
    P, I, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    fn = lib.slc_sparse_decode_static
    fn.restype = I
    fn.argtypes = [P, ctypes.POINTER(slc._Cache), P, I, P, I, I, I, I, I, F, P, P, P]
    return slc, fn


def _call_static(fn, slc, q, cache, bt, sl, P, W, K, out, sel):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(q.data_ptr(), cache.c, bt.data_ptr(), bt.shape[1], sl.data_ptr(), q.shape[0],
              q.shape[1], P, W, K, 0.0, out.data_ptr(), sel.data_ptr(), stream)


def test_static_scratch_decode_matches_workspace_decode_twice():
    slc, fn = _lib()
    # two different inputs, one after the other: the second call reuses the
    # scratch the first one left behind
    cases = [synth.make_inputs(synth.WORKLOADS["tiny"]),
             synth.make_inputs(synth.WORKLOADS["ragged"])]
    for x in cases:
        q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
        bt, sl = x.block_table.cuda(), x.seq_lens.cuda()
        cache = slc.PagedCache(k, v)
        slc.build_page_meta(cache, bt, sl)
        B, hkv = q.shape[0], k.shape[1]
        sel_ref = torch.empty((B, hkv, x.budget), dtype=torch.int32, device="cuda")
        ref = slc.sparse_decode(q, cache, bt, sl, x.prefix, x.window, x.budget,
                                selected_out=sel_ref)
        out = torch.full_like(ref, float("nan"))
        sel = torch.full_like(sel_ref, -7)
        rc = _call_static(fn, slc, q, cache, bt, sl, x.prefix, x.window, x.budget, out, sel)
        assert rc == 0, slc._lib.slc_error_string(rc)
        torch.cuda.synchronize()
        assert slc.device_status() == 0
        assert torch.equal(sel, sel_ref)
        err = (out - ref).abs().max().item()
        assert np.isfinite(err) and err <= OUT_TOL, err


def test_static_scratch_rejects_shapes_that_do_not_fit():
    slc, fn = _lib()
    need = slc._lib.slc_workspace_size(32, 32, 4, 128, 32768, 512)
    assert need > (16 << 20)
    q = torch.zeros((32, 32, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((32, 32768), dtype=torch.int32, device="cuda")
    sl = torch.zeros((32,), dtype=torch.int32, device="cuda")
    out = torch.empty((32, 32, 128), dtype=torch.float32, device="cuda")
    sel = torch.empty((32, 2, 512), dtype=torch.int32, device="cuda")
    cache4 = slc.PagedCache(torch.zeros((4, 4, 16, 128), dtype=torch.bfloat16, device="cuda"),
                            torch.zeros((4, 4, 16, 128), dtype=torch.bfloat16, device="cuda"))
    rc = _call_static(fn, slc, q, cache4, bt, sl, 0, 0, 512, out, sel)
    assert rc == -3  # SLC_ERR_WORKSPACE: nothing launched
