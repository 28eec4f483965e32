"""CUDA path against the fp64 oracle, element by element, on seeded inputs.

Bars: page metadata bit-exact; page selection identical except pages whose
oracle score is within 1e-4 (relative) of the k-th score; outputs within
2e-3 max-abs of the oracle attending the GPU's own selection."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import (Dev, check_needles, check_output, check_selection, oracle_scores,
                      slice_batch)

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def small(B, hq, hkv, D, lens, prefix=0, window=0, budget=0, layout="shuffled", seed=3,
          fill="zero", needles=0, headroom=0):
    wl = synth.Workload(name="t", batch=B, hq=hq, hkv=hkv, head_dim=D, prefix=prefix,
                        window=window, budget=budget, needles=needles, seed=seed,
                        context=max(lens), layout=layout)
    return synth.make_inputs(wl, lens_override=lens, fill=fill, headroom_tokens=headroom)


def meta_matches_oracle(d):
    x = d.x
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    meta = d.cache.meta.cpu().double().numpy()  # [pages][Hkv][2][D]
    bt = x.block_table.numpy()
    for b, L in enumerate(x.seq_lens.tolist()):
        n = -(-L // 16)
        phys = bt[b, :n]
        got_min = meta[phys, :, 0, :].transpose(1, 0, 2)  # [Hkv][n][D]
        got_max = meta[phys, :, 1, :].transpose(1, 0, 2)
        np.testing.assert_array_equal(got_min, kmin[b, :, :n])
        np.testing.assert_array_equal(got_max, kmax[b, :, :n])


@pytest.fixture(scope="module")
def tiny():
    return Dev(synth.make_inputs(W["tiny"]))


# ------------------------------------------------------------------ metadata

def test_build_page_meta_exact(tiny):
    meta_matches_oracle(tiny)


def test_build_page_meta_exact_ragged_lengths_nan_slots():
    x = small(5, 8, 4, 256, [1, 16, 17, 250, 1000], fill="nan", seed=7)
    meta_matches_oracle(Dev(x))


@pytest.mark.parametrize("hq,hkv,D", [(8, 2, 128), (16, 2, 256), (8, 8, 256)])
def test_kv_append_matches_rebuild_and_oracle(hq, hkv, D):
    """Appends across page boundaries (slot 0 resets a page's bounds) at both
    head dims: the cache holds the tokens where the host put them, and the
    incremental bounds equal the oracle's and a rebuild, bit for bit."""
    import sparse_long_context_max_b200 as slc
    x = small(3, hq, hkv, D, [30, 47, 16], seed=9 + D, headroom=40)
    d = Dev(x)
    lens = x.seq_lens.clone()
    for step in range(40):
        kn = torch.randn((3, hkv, D), generator=torch.Generator().manual_seed(step)).to(torch.bfloat16)
        vn = torch.randn((3, hkv, D), generator=torch.Generator().manual_seed(99 + step)).to(torch.bfloat16)
        slc.kv_append(d.cache, kn.cuda(), vn.cuda(), d.bt, lens.cuda())
        for b in range(3):
            L = int(lens[b])
            phys = int(x.block_table[b, L // 16])
            x.k_cache[phys, :, L % 16] = kn[b]
            x.v_cache[phys, :, L % 16] = vn[b]
        lens += 1
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    # the appended tokens landed where the host put them
    assert torch.equal(d.k.cpu(), x.k_cache)
    assert torch.equal(d.v.cpu(), x.v_cache)
    x.seq_lens = lens
    d.sl = lens.cuda()
    incremental = d.cache.meta.clone()
    meta_matches_oracle(d)
    slc.build_page_meta(d.cache, d.bt, d.sl)
    rebuilt = d.cache.meta
    used = sorted(set(int(p) for b in range(3) for p in x.block_table[b, : -(-int(lens[b]) // 16)]))
    assert torch.equal(incremental[used].float(), rebuilt[used].float())


# ------------------------------------------------------------------ scoring

def test_scores_match_oracle_and_bound(tiny):
    import sparse_long_context_max_b200 as slc
    x = tiny.x
    s = slc.score_pages(tiny.q, tiny.cache, tiny.bt, tiny.sl, x.prefix, x.window).cpu().double().numpy()
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    so = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, x.prefix, x.window)
    cand = ~np.isnan(so)
    assert cand.sum() == 2 * (240 - 4)
    scale = np.abs(so[cand]).max()
    assert np.abs(s[cand] - so[cand]).max() <= 2e-6 * scale
    # the bound never drops below the best group logit of the page
    G = 4
    for h in range(2):
        for j in range(4, 240):
            phys = int(x.block_table[0, j])
            k = x.k_cache[phys, h].double()
            q = x.q[0, h * G:(h + 1) * G].double()
            best = (q @ k.T).sum(0).max().item()
            assert s[0, h, j] >= best - 1e-5 * abs(best) - 1e-4


def stream_scores(d, prefix, window, budget):
    """The candidate scores the sparse decode itself computes (its streaming
    kernel, stage 1), read back from the workspace: float64
    [B][Hkv][max_pages] by page, NaN outside the candidates."""
    import sparse_long_context_max_b200 as slc
    x = d.x
    B, hq, D = x.q.shape
    hkv = x.k_cache.shape[1]
    mp = x.block_table.shape[1]
    ws = torch.zeros(slc.workspace_size(B, hq, hkv, D, mp, budget), dtype=torch.uint8,
                     device="cuda")
    slc.sparse_decode_stage(1, d.q, d.cache, d.bt, d.sl, prefix, window, budget, workspace=ws)
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    cs = (mp + 63) // 64 * 64  # rows by candidate, 64-float aligned
    rows = ws[: B * hkv * cs * 4].view(torch.float32).view(B, hkv, cs).cpu().double().numpy()
    out = np.full((B, hkv, mp), np.nan)
    for b, L in enumerate(x.seq_lens.tolist()):
        n, np_, wsp = oracle.page_ranges(L, prefix, window)
        out[b, :, np_:wsp] = rows[b, :, : wsp - np_]
    return out


def check_scores(x, s, prefix, window, rel=2e-6):
    """GPU scores within rel (of the largest score) of the oracle's, and never
    below the oracle's own best group logit of a sampled page."""
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    so = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, prefix, window)
    cand = ~np.isnan(so)
    assert (np.isnan(s) == ~cand).all()
    scale = np.abs(so[cand]).max()
    assert np.abs(s[cand] - so[cand]).max() <= rel * scale
    return so


def test_stream_scores_match_oracle_decode256k():
    """The decode path's own scores at 256k (group 8, d 128): every candidate
    of every unit within 2e-6 (relative) of the oracle."""
    x = synth.make_inputs(W["decode256k"])
    d = Dev(x)
    check_scores(x, stream_scores(d, x.prefix, x.window, x.budget), x.prefix, x.window)


def test_stream_scores_match_oracle_layers131k():
    """The same at d 256 (one layer of the 131k plan, group 8)."""
    wl = W["layers131k"]
    plan = synth.layer_plan(wl)
    layer = [i for i, (_, _, dn) in enumerate(plan) if not dn][0]
    x = synth.make_inputs(wl, layer=layer)
    d = Dev(x)
    check_scores(x, stream_scores(d, x.prefix, x.window, x.budget), x.prefix, x.window)


def test_select_exact_on_given_scores():
    import sparse_long_context_max_b200 as slc
    rng = np.random.default_rng(0)
    for ncand, budget, ties in [(50, 7, True), (4000, 128, True), (16120, 256, False),
                                (16120, 256, True), (30000, 512, True), (9, 3, True)]:
        B, hkv = 2, 3
        L = 16 * (ncand + 2)
        P, Wn = 16, 16
        scores = np.full((B, hkv, ncand + 2), np.nan, dtype=np.float32)
        if ties:
            vals = rng.integers(-20, 20, size=(B, hkv, ncand)).astype(np.float32)
        else:
            vals = rng.standard_normal((B, hkv, ncand)).astype(np.float32) * 100
        scores[:, :, 1:ncand + 1] = vals
        sl = torch.tensor([L, L], dtype=torch.int32)
        sel = slc.select_pages(torch.from_numpy(scores).cuda(), sl.cuda(), P, Wn, budget)
        want, _ = oracle.select_pages(scores.astype(np.float64), sl, P, Wn, budget)
        np.testing.assert_array_equal(sel.cpu().numpy(), want)


# ------------------------------------------------------------------ decode

def test_tiny_sparse_parity(tiny):
    x = tiny.x
    out, sel = tiny.sparse()
    check_selection(x, sel, x.prefix, x.window, x.budget)
    check_needles(x, sel)
    check_output(x, out, x.prefix, x.window, sel)


def test_sparse_attend_with_another_layers_selection():
    """Cross-layer reuse of a selection ("IndexCache: cross-layer reuse speeds
    30B prefill 1.82x": a Shared layer takes the indices of the preceding
    Full layer): slc_sparse_attend, given a selection and another query,
    attends the prefix, the window and exactly the given pages."""
    import copy
    import sparse_long_context_max_b200 as slc
    # the short sequence has fewer candidates than the budget: -1 padding
    x = small(3, 16, 4, 128, [5000, 2100, 900], prefix=64, window=256, budget=40, seed=21)
    d = Dev(x)
    _, sel = d.sparse()  # the Full layer's selection
    q2 = torch.randn(x.q.shape, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    out = slc.sparse_attend(q2.cuda(), d.cache, d.bt, d.sl, x.prefix, x.window,
                            torch.from_numpy(sel).cuda())
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    assert (sel[2] == -1).any()
    y = copy.copy(x)
    y.q = q2
    check_output(y, out.cpu().double().numpy(), x.prefix, x.window, sel)


def test_sparse_attend_union_semantics():
    """A given selection is attended as a set united with the prefix and
    window: entries that are prefix or window pages add nothing, -1 is
    padding, and out-of-range or out-of-order entries are skipped and
    flagged.  Compared with the oracle, whose attended set is that union."""
    import sparse_long_context_max_b200 as slc
    x = small(2, 8, 2, 128, [3000, 1000], prefix=32, window=128, budget=8, seed=31)
    d = Dev(x)
    n0, np0, ws0 = oracle.page_ranges(3000, 32, 128)
    n1, np1, ws1 = oracle.page_ranges(1000, 32, 128)
    sel = np.full((2, 2, 8), -1, dtype=np.int32)
    sel[0, 0, :6] = [0, 5, 40, 100, ws0, n0 - 1]  # prefix, candidates, window pages
    sel[0, 1, :3] = [7, 9, 11]
    sel[1, 0, :4] = [3, 4, ws1 + 1, n1 - 1]
    sel[1, 1, :2] = [np1, ws1 - 1]
    out = slc.sparse_attend(d.q, d.cache, d.bt, d.sl, 32, 128, torch.from_numpy(sel).cuda())
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    check_output(x, out.cpu().double().numpy(), 32, 128, sel)
    bad = sel.copy()
    bad[0, 0, 6] = n0 + 5  # past the sequence
    bad[1, 1, 2] = 1  # not above the entry before it
    out2 = slc.sparse_attend(d.q, d.cache, d.bt, d.sl, 32, 128, torch.from_numpy(bad).cuda())
    torch.cuda.synchronize()
    assert slc.device_status() & 4  # bad selection, skipped
    check_output(x, out2.cpu().double().numpy(), 32, 128, sel)


@pytest.mark.parametrize("lens,budget", [([5000, 9000, 700], 37), ([262144 // 8, 3000], 300)])
def test_selection_ties_go_to_the_lower_page(lens, budget):
    """Keys of +-1 only: nearly every page has the bounds (-1, +1) in every
    dimension, so nearly every candidate has the same score, computed the
    same way on the GPU.  The selection must then be the lowest-indexed of
    the top-scoring pages, exactly: the tie-break of the method's total
    order, exercised across all CTAs of a cluster."""
    x = small(len(lens), 8, 2, 128, lens, prefix=64, window=256, budget=budget, seed=41)
    x.k_cache = torch.where(x.k_cache >= 0, 1.0, -1.0).to(torch.bfloat16)
    d = Dev(x)
    out, sel = d.sparse()
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    so = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, x.prefix, x.window)
    want, _ = oracle.select_pages(so, x.seq_lens, x.prefix, x.window, budget)
    np.testing.assert_array_equal(sel, want)
    check_output(x, out, x.prefix, x.window, sel)


def test_stages_in_order_equal_one_call():
    """slc_sparse_decode_stage 1 then 2 on one workspace reproduce
    slc_sparse_decode bit for bit (same kernels, same order)."""
    import sparse_long_context_max_b200 as slc
    x = synth.make_inputs(W["ragged"])
    d = Dev(x)
    B, hq, D = x.q.shape
    hkv = x.k_cache.shape[1]
    ws = torch.zeros(slc.workspace_size(B, hq, hkv, D, x.block_table.shape[1], x.budget),
                     dtype=torch.uint8, device="cuda")
    sel1 = torch.empty((B, hkv, x.budget), dtype=torch.int32, device="cuda")
    sel2 = torch.full_like(sel1, -7)
    out1 = slc.sparse_decode(d.q, d.cache, d.bt, d.sl, x.prefix, x.window, x.budget,
                             selected_out=sel1, workspace=ws)
    out2 = torch.full_like(out1, float("nan"))
    ws.zero_()
    for stage in (1, 2):
        slc.sparse_decode_stage(stage, d.q, d.cache, d.bt, d.sl, x.prefix, x.window, x.budget,
                                out=out2, selected_out=sel2, workspace=ws)
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    assert torch.equal(sel1, sel2)
    assert torch.equal(out1, out2)
    for bad in (0, 3, -1):
        with pytest.raises(slc.SLCError):
            slc.sparse_decode_stage(bad, d.q, d.cache, d.bt, d.sl, x.prefix, x.window, x.budget,
                                    out=out2, selected_out=sel2, workspace=ws)


def test_tiny_dense_parity(tiny):
    check_output(tiny.x, tiny.dense(), 0, 0, None, dense=True)


def test_coverage_equals_dense(tiny):
    x = tiny.x
    dense = tiny.dense()
    out, sel = tiny.sparse(budget=400)
    assert (sel[0, :, :236] >= 0).all()
    assert np.abs(out - dense).max() <= 1e-5
    check_output(x, out, x.prefix, x.window, None, dense=True)


def test_budget_zero(tiny):
    x = tiny.x
    out, _ = tiny.sparse(budget=0)
    check_output(x, out, x.prefix, x.window, np.full((1, 2, 0), -1, dtype=np.int32))


def test_nan_sentinels_do_not_leak():
    a = small(4, 8, 2, 128, [37, 600, 16, 1201], prefix=20, window=100, budget=5, fill="zero")
    b = small(4, 8, 2, 128, [37, 600, 16, 1201], prefix=20, window=100, budget=5, fill="nan")
    oa, sa = Dev(a).sparse()
    ob, sb = Dev(b).sparse()
    np.testing.assert_array_equal(sa, sb)
    np.testing.assert_array_equal(oa, ob)
    check_output(b, ob, 20, 100, sb)


def test_layout_invariance():
    a = small(3, 8, 2, 128, [900, 333, 2000], prefix=32, window=64, budget=6, layout="contiguous")
    b = small(3, 8, 2, 128, [900, 333, 2000], prefix=32, window=64, budget=6, layout="shuffled")
    oa, sa = Dev(a).sparse()
    ob, sb = Dev(b).sparse()
    np.testing.assert_array_equal(sa, sb)
    assert np.abs(oa - ob).max() <= 1e-6


@pytest.mark.parametrize("hq,hkv,D", [(8, 2, 128), (4, 4, 128), (6, 2, 128), (16, 2, 256),
                                      (8, 8, 256)])
def test_edge_lengths_and_groups(hq, hkv, D):
    lens = [0, 1, 15, 16, 17, 33, 100, 257, 1999]
    x = small(len(lens), hq, hkv, D, lens, seed=hq * 31 + D, fill="nan")
    d = Dev(x)
    meta_matches_oracle(d)
    for P, Wn, K in [(0, 0, 3), (16, 32, 2), (5, 1, 0), (64, 256, 100), (0, 16, 1)]:
        out, sel = d.sparse(P, Wn, K)
        check_selection(x, sel, P, Wn, K)
        check_output(x, out, P, Wn, sel)
        assert (out[0] == 0).all()  # empty sequence
    check_output(x, d.dense(), 0, 0, None, dense=True)


def test_explicit_scale(tiny):
    x = tiny.x
    out, sel = tiny.sparse(scale=0.3)
    want = oracle.attend(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, x.prefix,
                         x.window, sel, scale=0.3)
    assert np.abs(out - want).max() <= 2e-3


def test_bad_block_table_entry_is_flagged_not_followed():
    import sparse_long_context_max_b200 as slc
    x = small(2, 8, 2, 128, [300, 300], prefix=16, window=32, budget=4)
    d = Dev(x)
    bt = d.bt.clone()
    bt[1, 5] = x.k_cache.shape[0] + 1000  # outside the pool
    bt[0, 7] = -3
    slc.sparse_decode(d.q, d.cache, bt, d.sl, 16, 32, 4)
    torch.cuda.synchronize()
    st = slc.device_status()
    assert st & 1  # bad page
    assert slc.device_status() == 0  # cleared
    bad_len = d.sl.clone()
    bad_len[0] = 10 ** 6
    slc.dense_decode(d.q, d.cache, d.bt, bad_len)
    torch.cuda.synchronize()
    assert slc.device_status() & 2


# ------------------------------------------------------------------ workloads

def test_ragged_workload_parity():
    x = synth.make_inputs(W["ragged"], fill="nan")
    d = Dev(x)
    out, sel = d.sparse()
    check_selection(x, sel, x.prefix, x.window, x.budget)
    check_needles(x, sel)
    check_output(x, out, x.prefix, x.window, sel)
    # the two short sequences are covered whole: equal to dense attention
    dense = d.dense()
    assert np.abs(out[:2] - dense[:2]).max() <= 1e-5
    check_output(x, dense, 0, 0, None, dense=True)  # every sequence


def test_decode256k_parity():
    x = synth.make_inputs(W["decode256k"])
    d = Dev(x)
    out, sel = d.sparse()
    check_selection(x, sel, x.prefix, x.window, x.budget)
    check_needles(x, sel)
    check_output(x, out, x.prefix, x.window, sel)
    dense = d.dense()
    check_output(x, dense, 0, 0, None, dense=True)  # every sequence


def test_decode64k_append_loop():
    import sparse_long_context_max_b200 as slc
    wl = W["decode64k"]
    x = synth.make_inputs(wl)
    d = Dev(x)
    lens = x.seq_lens.clone()
    check_at = {0, 1, 17, wl.steps - 1}
    for step in range(wl.steps):
        if step > 0:
            q, kn, vn = synth.step_tokens(wl, step)
            # append the new token, then decode with it in the context
            slc.kv_append(d.cache, kn.cuda(), vn.cuda(), d.bt, lens.cuda())
            for b in range(wl.batch):
                L = int(lens[b])
                phys = int(x.block_table[b, L // 16])
                x.k_cache[phys, :, L % 16] = kn[b]
                x.v_cache[phys, :, L % 16] = vn[b]
            lens += 1
            x.q = q
            d.q = q.cuda()
            x.seq_lens = lens.clone()
            d.sl = lens.cuda()
        if step in check_at:
            out, sel = d.sparse()
            check_selection(x, sel, x.prefix, x.window, x.budget)
            if step == 0:
                check_needles(x, sel)
            check_output(x, out, x.prefix, x.window, sel)
        else:
            import sparse_long_context_max_b200 as s2
            s2.sparse_decode(d.q, d.cache, d.bt, d.sl, x.prefix, x.window, x.budget)
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    incremental = d.cache.meta.clone()
    slc.build_page_meta(d.cache, d.bt, d.sl)
    used = x.block_table[:, : -(-int(lens.max()) // 16)].reshape(-1).long()
    assert torch.equal(incremental[used.cuda()].float(), d.cache.meta[used.cuda()].float())


def test_layers131k_sampled_layers():
    wl = W["layers131k"]
    plan = synth.layer_plan(wl)
    dense_layer = [i for i, (_, _, dn) in enumerate(plan) if dn][0]
    sparse_layers = [i for i, (_, _, dn) in enumerate(plan) if not dn][:2]
    for layer in sparse_layers + [dense_layer]:
        x = synth.make_inputs(wl, layer=layer)
        d = Dev(x)
        if plan[layer][2]:
            out = d.dense()
            check_output(x, out, 0, 0, None, dense=True)  # every sequence
        else:
            out, sel = d.sparse()
            check_selection(x, sel, x.prefix, x.window, x.budget)
            check_needles(x, sel)
            check_output(x, out, x.prefix, x.window, sel)
        del d, x
        torch.cuda.empty_cache()


def test_layers131k_graph_step_all_layers():
    """One decode step of the 15-layer plan at 131072 tokens (d 256), replayed
    from its CUDA graph with the inputs copied in from pinned host buffers
    and the outputs copied back: per layer the new token's append, then the
    layer's decode.  Cross-layer reuse is on ("IndexCache: cross-layer reuse speeds
    30B prefill 1.82x": Full layers select, Shared layers attend the nearest
    Full layer's selection with their own window).  Checked per layer: the
    appended token landed, Full layers' selections against the oracle's
    (tie band), every sparse layer's output against the oracle attending
    prefix + window + the selection it used, the dense layers on every
    sequence."""
    import sparse_long_context_max_b200 as slc
    from sparse_long_context_max_b200 import plan as P
    wl = W["layers131k"]
    x = synth.make_inputs(wl, layer=0, headroom_tokens=16)
    layers = synth.layer_plan(wl)
    specs = P.index_reuse([P.LayerSpec(w, k, dn) for w, k, dn in layers])
    assert any(s.shared for s in specs) and any(s.dense for s in specs)
    k0, v0 = x.k_cache.cuda(), x.v_cache.cuda()
    bt = x.block_table.cuda()
    caches = []
    for _ in specs:
        c = slc.PagedCache(k0.clone(), v0.clone())
        slc.build_page_meta(c, bt, x.seq_lens.cuda())
        caches.append(c)
    del k0, v0
    step = P.DecodeStep(caches, bt, specs, wl.prefix, wl.hq)
    toks = [synth.step_tokens(wl, 1, layer=i) for i in range(len(specs))]
    io = step.host_buffers()  # the inputs travel as one packed host-to-device copy
    for i, (q, kn, vn) in enumerate(toks):
        io.q[i].copy_(q)
        io.k_new[i].copy_(kn)
        io.v_new[i].copy_(vn)
    io.positions.copy_(x.seq_lens)
    io.seq_lens.copy_(x.seq_lens + 1)
    step.run_from_host(io)  # captures on first use, then replays
    step.run_from_host(io)  # the append writes the same slot again: idempotent
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    assert torch.equal(io.out, step.out.cpu())
    lens1 = x.seq_lens + 1
    for i, s in enumerate(specs):
        q, kn, vn = toks[i]
        y = slice_batch(x, list(range(wl.batch)))
        y.q, y.seq_lens = q, lens1
        y.k_cache, y.v_cache = x.k_cache.clone(), x.v_cache.clone()
        for b in range(wl.batch):
            L = int(x.seq_lens[b])
            phys = int(x.block_table[b, L // 16])
            y.k_cache[phys, :, L % 16] = kn[b]
            y.v_cache[phys, :, L % 16] = vn[b]
        got = caches[i]
        for b in range(wl.batch):
            L = int(x.seq_lens[b])
            phys = int(x.block_table[b, L // 16])
            assert torch.equal(got.k_cache[phys, :, L % 16].cpu(), kn[b])
        out = step.out[i].cpu().double().numpy()
        if s.dense:
            check_output(y, out, 0, 0, None, dense=True)  # every sequence
            continue
        if not s.shared:
            sel = step.selected[i].cpu().numpy()
            check_selection(y, sel, wl.prefix, s.window, s.budget)
        else:
            sel = step.selected[step.full_of[i]].cpu().numpy()
        check_output(y, out, wl.prefix, s.window, sel)
    del caches, step
    torch.cuda.empty_cache()



# ------------------------------------------------------------------ E4M3 metadata

def meta8_matches_oracle(d):
    """The device's E4M3 bounds equal the oracle's outward-rounded codes,
    bit for bit."""
    x = d.x
    c8min, c8max = oracle.page_bounds_fp8(x.k_cache, x.block_table, x.seq_lens)
    meta = d.cache.meta.cpu().numpy()  # uint8 [pages][Hkv][2][D]
    bt = x.block_table.numpy()
    for b, L in enumerate(x.seq_lens.tolist()):
        n = -(-L // 16)
        phys = bt[b, :n]
        np.testing.assert_array_equal(meta[phys, :, 0, :].transpose(1, 0, 2), c8min[b, :, :n])
        np.testing.assert_array_equal(meta[phys, :, 1, :].transpose(1, 0, 2), c8max[b, :, :n])


@pytest.mark.parametrize("hq,hkv,D", [(8, 2, 128), (16, 2, 256)])
def test_fp8_meta_build_and_append_exact(hq, hkv, D):
    """E4M3 metadata, built and appended: bit-exact against the oracle's
    outward rounding, keys spread from subnormal E4M3 to beyond +-448 and
    NaN/Inf in unused slots; the appended form equals a rebuild."""
    import sparse_long_context_max_b200 as slc
    x = small(3, hq, hkv, D, [30, 47, 16], seed=23 + D, headroom=40, fill="nan")
    g = torch.Generator().manual_seed(5)
    scale = torch.exp(torch.randn(x.k_cache.shape, generator=g) * 3)  # e^-9 .. e^9
    x.k_cache = torch.where(torch.isfinite(x.k_cache.float()),
                            x.k_cache.float() * scale, x.k_cache.float()).to(torch.bfloat16)
    d = Dev(x, meta_format="fp8")
    meta8_matches_oracle(d)
    lens = x.seq_lens.clone()
    for step in range(40):
        kn = (torch.randn((3, hkv, D), generator=torch.Generator().manual_seed(step)) *
              torch.exp(torch.randn((3, hkv, D), generator=g) * 3)).to(torch.bfloat16)
        vn = torch.randn((3, hkv, D), generator=torch.Generator().manual_seed(77 + step)).to(torch.bfloat16)
        slc.kv_append(d.cache, kn.cuda(), vn.cuda(), d.bt, lens.cuda())
        for b in range(3):
            L = int(lens[b])
            phys = int(x.block_table[b, L // 16])
            x.k_cache[phys, :, L % 16] = kn[b]
            x.v_cache[phys, :, L % 16] = vn[b]
        lens += 1
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    x.seq_lens = lens
    d.sl = lens.cuda()
    incremental = d.cache.meta.clone()
    meta8_matches_oracle(d)
    slc.build_page_meta(d.cache, d.bt, d.sl)
    used = sorted(set(int(p) for b in range(3) for p in x.block_table[b, : -(-int(lens[b]) // 16)]))
    assert torch.equal(incremental[used], d.cache.meta[used])


@pytest.mark.parametrize("name", ["tiny", "decode256k"])
def test_fp8_meta_decode_parity(name):
    """Sparse decode over E4M3 metadata: the decode path's own scores against
    the oracle's scores from the outward-rounded bounds (2e-6 relative), the
    selection within the tie band of those scores, the output against the
    oracle attending the GPU's selection, and needles still selected."""
    x = synth.make_inputs(W[name])
    d = Dev(x, meta_format="fp8")
    so = oracle_scores(x, x.prefix, x.window, "fp8")
    s = stream_scores(d, x.prefix, x.window, x.budget)
    cand = ~np.isnan(so)
    assert (np.isnan(s) == ~cand).all()
    assert np.abs(s[cand] - so[cand]).max() <= 2e-6 * np.abs(so[cand]).max()
    out, sel = d.sparse()
    check_selection(x, sel, x.prefix, x.window, x.budget, scores=so)
    check_needles(x, sel)
    check_output(x, out, x.prefix, x.window, sel)


# ------------------------------------------------------------------ top-delta

def test_select_delta_exact_on_given_scores():
    """Top-delta selection kernel against the oracle on scores of a 0.25 grid
    (exact in fp32, so the fp32 threshold s_max - delta equals the oracle's):
    bit-exact, over ties, caps below and above the union, d = 0, a negative
    and an infinite delta, and unit sizes on both of the kernel's paths."""
    import sparse_long_context_max_b200 as slc
    rng = np.random.default_rng(12)
    for ncand, d, delta, cap in [(50, 7, 1.0, 20), (50, 7, 1.0, 3), (4000, 128, 0.5, 300),
                                 (16120, 256, 2.0, 512), (16120, 0, 0.75, 64),
                                 (16120, 16, -1.0, 64), (900, 4, float("inf"), 1000),
                                 (30000, 200, 1.5, 700), (9, 3, 0.25, 9)]:
        B, hkv = 2, 3
        L = 16 * (ncand + 2)
        scores = np.full((B, hkv, ncand + 2), np.nan, dtype=np.float32)
        scores[:, :, 1:ncand + 1] = np.round(rng.standard_normal((B, hkv, ncand)) * 8) / 4
        sl = torch.tensor([L, L], dtype=torch.int32)
        sel = slc.select_pages_delta(torch.from_numpy(scores).cuda(), sl.cuda(), 16, 16, d,
                                     delta, cap)
        want, _ = oracle.select_pages_delta(scores.astype(np.float64), sl, 16, 16, d, delta, cap)
        np.testing.assert_array_equal(sel.cpu().numpy(), want, err_msg=str((ncand, d, delta, cap)))


def check_selection_delta(x, sel_gpu, d, delta, cap, scores):
    """GPU top-delta selection == the oracle's, except pages whose oracle
    score is within TIE_BAND (relative to the best score) of one of the two
    boundaries: the d-th best score and s_max - delta."""
    sel_o, nsel_o = oracle.select_pages_delta(scores, x.seq_lens, x.prefix, x.window, d, delta,
                                              cap)
    B, hkv, _ = sel_o.shape
    for b in range(B):
        n, np_, ws = oracle.page_ranges(int(x.seq_lens[b]), x.prefix, x.window)
        for h in range(hkv):
            cand = scores[b, h, np_:ws]
            smax = float(cand.max())
            order = np.sort(cand)[::-1]
            dth = float(order[min(d, len(order)) - 1]) if d > 0 else smax
            o = set(int(p) for p in sel_o[b, h] if p >= 0)
            g = [int(p) for p in sel_gpu[b, h]]
            k = len([p for p in g if p >= 0])
            assert g[k:] == [-1] * (cap - k) and g[:k] == sorted(g[:k]), (b, h)
            for p in o ^ set(g[:k]):
                s = scores[b, h, p]
                near = min(abs(s - dth), abs(s - (smax - delta)))
                assert near <= TIE_BAND * abs(smax), (b, h, p, s, smax)


@pytest.mark.parametrize("d,delta,cap", [(8, 3.0, 64), (8, 3.0, 6), (0, -1.0, 32), (5, 0.0, 40),
                                         (0, float("inf"), 300), (400, 1.0, 500), (3, 1e30, 20),
                                         (16, 6.0, 0)])
def test_sparse_decode_delta_matches_the_standalone_selection(d, delta, cap):
    """The top-delta decode step sets each unit's selection size inside the
    finishing kernel; on the same scores (the scoring code is shared) its
    selection equals the standalone top-delta kernel's bit for bit, over the
    edges: d past the candidates, cap below d, nothing within a negative
    delta of the best with d = 0, every candidate (delta = inf), cap 0.  The
    output is checked against the oracle attending that selection."""
    import sparse_long_context_max_b200 as slc
    x = small(3, 8, 2, 128, [4096, 2000, 300], prefix=32, window=256, seed=41, needles=4)
    dv = Dev(x)
    B, hq, D = x.q.shape
    hkv = x.k_cache.shape[1]
    width = max(cap, 1)
    sel = torch.full((B, hkv, width), -7, dtype=torch.int32, device="cuda")[:, :, :cap]
    sel = sel.contiguous()
    out = slc.sparse_decode_delta(dv.q, dv.cache, dv.bt, dv.sl, x.prefix, x.window, d, delta,
                                  cap, selected_out=sel if cap > 0 else None)
    scores = slc.score_pages(dv.q, dv.cache, dv.bt, dv.sl, x.prefix, x.window)
    want = slc.select_pages_delta(scores, dv.sl, x.prefix, x.window, d, delta, cap) \
        if cap > 0 else torch.empty((B, hkv, 0), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    np.testing.assert_array_equal(sel.cpu().numpy(), want.cpu().numpy())
    check_output(x, out.cpu().double().numpy(), x.prefix, x.window, sel.cpu().numpy())


@pytest.mark.parametrize("name,d,delta,cap", [("tiny", 8, 2.0, 64), ("decode256k", 64, 40.0, 512),
                                              ("ragged", 16, 25.0, 128)])
def test_sparse_decode_delta_parity(name, d, delta, cap):
    """The top-delta decode step (scores, top-delta selection, attention over
    prefix + window + selection): the selection against the oracle's on the
    oracle's scores within the tie bands, every needle page selected, and
    the output against the oracle attending the GPU's selection."""
    import sparse_long_context_max_b200 as slc
    x = synth.make_inputs(W[name], fill="nan" if name == "ragged" else "zero")
    dv = Dev(x)
    B, hq, D = x.q.shape
    hkv = x.k_cache.shape[1]
    sel = torch.full((B, hkv, cap), -7, dtype=torch.int32, device="cuda")
    out = slc.sparse_decode_delta(dv.q, dv.cache, dv.bt, dv.sl, x.prefix, x.window, d, delta,
                                  cap, selected_out=sel)
    torch.cuda.synchronize()
    assert slc.device_status() == 0
    sel = sel.cpu().numpy()
    so = oracle_scores(x, x.prefix, x.window)
    check_selection_delta(x, sel, d, delta, cap, so)
    if name != "ragged":  # the needle pages top the scores: within the top d
        check_needles(x, sel)
    check_output(x, out.cpu(), x.prefix, x.window, sel)
