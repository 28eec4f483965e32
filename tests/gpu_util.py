"""Helpers shared by the GPU parity tests: device copies of the synthetic
inputs, calls through the binding, and the oracle comparisons."""
import numpy as np
import torch

import oracle

OUT_TOL = 2e-3  # max-abs output error against the fp64 oracle
TIE_BAND = 1e-4  # selections may differ only on pages this close to the k-th score


class Dev:
    """Device copies of one layer's inputs, plus the cache object."""

    def __init__(self, x, build_meta=True, meta_format="bf16"):
        import sparse_long_context_max_b200 as slc
        self.x = x
        self.q = x.q.cuda()
        self.k = x.k_cache.cuda()
        self.v = x.v_cache.cuda()
        self.bt = x.block_table.cuda()
        self.sl = x.seq_lens.cuda()
        self.meta_format = meta_format
        self.cache = slc.PagedCache(self.k, self.v, meta_format=meta_format)
        if build_meta:
            slc.build_page_meta(self.cache, self.bt, self.sl)

    def sparse(self, prefix=None, window=None, budget=None, scale=0.0):
        import sparse_long_context_max_b200 as slc
        x = self.x
        P = x.prefix if prefix is None else prefix
        W = x.window if window is None else window
        K = x.budget if budget is None else budget
        B, hkv = self.q.shape[0], self.k.shape[1]
        sel = torch.full((B, hkv, max(K, 1)), -7, dtype=torch.int32, device="cuda")[:, :, :K]
        sel = sel.contiguous()
        out = slc.sparse_decode(self.q, self.cache, self.bt, self.sl, P, W, K, scale=scale,
                                selected_out=sel if K > 0 else None)
        torch.cuda.synchronize()
        assert slc.device_status() == 0
        return out.cpu().double().numpy(), sel.cpu().numpy()

    def dense(self, scale=0.0):
        import sparse_long_context_max_b200 as slc
        out = slc.dense_decode(self.q, self.cache, self.bt, self.sl, scale=scale)
        torch.cuda.synchronize()
        assert slc.device_status() == 0
        return out.cpu().double().numpy()


def oracle_scores(x, prefix, window, meta_format="bf16"):
    """The oracle's page scores from bf16 bounds, or from the E4M3 bounds
    rounded outward."""
    if meta_format == "fp8":
        c8min, c8max = oracle.page_bounds_fp8(x.k_cache, x.block_table, x.seq_lens)
        kmin, kmax = oracle.fp8_decode(c8min), oracle.fp8_decode(c8max)
    else:
        kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    return oracle.page_scores(x.q, kmin, kmax, x.seq_lens, prefix, window)


def check_selection(x, sel_gpu, prefix, window, budget, scores=None, meta_format="bf16"):
    """GPU selection == oracle selection, except pages whose oracle score is
    within TIE_BAND (relative) of the k-th oracle score.  Returns the oracle
    selection."""
    if scores is None:
        scores = oracle_scores(x, prefix, window, meta_format)
    sel_o, nsel_o = oracle.select_pages(scores, x.seq_lens, prefix, window, budget)
    B, hkv, _ = sel_o.shape
    for b in range(B):
        for h in range(hkv):
            o = set(int(p) for p in sel_o[b, h] if p >= 0)
            g = [int(p) for p in sel_gpu[b, h]]
            n = int(nsel_o[b, h])
            assert g[n:] == [-1] * (budget - n), (b, h, "padding")
            assert g[:n] == sorted(g[:n]), (b, h, "not ascending")
            g = set(g[:n])
            assert len(g) == n
            if o == g:
                continue
            kth = min(scores[b, h, p] for p in o)
            for p in o ^ g:
                assert abs(scores[b, h, p] - kth) <= TIE_BAND * abs(kth), (b, h, p)
    return sel_o


def check_output(x, out_gpu, prefix, window, sel_gpu, dense=False, tol=OUT_TOL):
    """Output within tol of the fp64 oracle attending the GPU's own
    selection (or every token when dense)."""
    want = oracle.attend(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, prefix, window,
                         None if dense else sel_gpu, dense=dense)
    err = np.abs(out_gpu - want).max() if want.size else 0.0
    assert np.isfinite(out_gpu).all()
    assert err <= tol, err
    return err


def check_needles(x, sel_gpu):
    B, hkv, _ = sel_gpu.shape
    for b in range(B):
        for h in range(hkv):
            chosen = set(sel_gpu[b, h].tolist())
            for t in x.needle_tokens[b]:
                assert t // 16 in chosen, (b, h, t)


def slice_batch(x, bs):
    """A copy of the inputs restricted to the sequences in bs."""
    import copy
    y = copy.copy(x)
    idx = torch.tensor(bs, dtype=torch.long)
    y.q = x.q[idx].contiguous()
    y.block_table = x.block_table[idx].contiguous()
    y.seq_lens = x.seq_lens[idx].contiguous()
    y.needle_tokens = [x.needle_tokens[b] for b in bs]
    return y
