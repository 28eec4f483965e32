"""Pins for the CPU oracle: hand-worked fixtures, closed forms, library
special cases, invariants and brute force.  CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import GOLDEN


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16(x):
    t = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(x, dtype=torch.float32)), "not bf16-exact"
    return t


def _small_cache(B, Hq, Hkv, D, lens, layout="shuffled", seed=5, fill="zero"):
    wl = synth.Workload(name="t", batch=B, hq=Hq, hkv=Hkv, head_dim=D, prefix=0,
                        window=0, budget=0, needles=0, seed=seed, context=max(lens),
                        layout=layout)
    return synth.make_inputs(wl, lens_override=lens, fill=fill, threads=1)


# ---------------------------------------------------------------- fixtures

def test_page_ranges_golden():
    for c in _load("page_ranges.json")["cases"]:
        assert oracle.page_ranges(c["L"], c["P"], c["W"]) == (c["n"], c["np"], c["ws"]), c


def test_score_golden():
    g = _load("score_example.json")
    q = _bf16(g["q"]).reshape(1, 2, 2)
    kmin = np.array(g["kmin"], dtype=np.float64).reshape(1, 1, 3, 2)
    kmax = np.array(g["kmax"], dtype=np.float64).reshape(1, 1, 3, 2)
    s = oracle.page_scores(q, kmin, kmax, [48], prefix=0, window=0)
    assert s[0, 0].tolist() == g["scores"]


def test_select_golden():
    g = _load("select_example.json")
    # L = 176 tokens (11 pages), prefix 32 -> pages 0,1; window 16 -> page 10
    L, P, W = 176, 32, 16
    assert oracle.page_ranges(L, P, W)[1:] == (g["np"], g["ws"])
    scores = np.full((1, 1, 11), np.nan)
    for j, v in g["scores"].items():
        scores[0, 0, int(j)] = v
    for c in g["cases"]:
        sel, nsel = oracle.select_pages(scores, [L], P, W, c["budget"])
        got = [int(x) for x in sel[0, 0] if x >= 0]
        assert got == c["sel"], c
        assert nsel[0, 0] == len(c["sel"])


def test_attend_golden():
    g = _load("attend_example.json")
    D = 2
    k = torch.zeros((1, 1, 16, D), dtype=torch.bfloat16)
    v = torch.zeros((1, 1, 16, D), dtype=torch.bfloat16)
    k[0, 0, :2] = _bf16(g["k"])
    v[0, 0, :2] = _bf16(g["v"])
    q = _bf16(g["q"]).reshape(1, 1, D)
    out = oracle.dense_decode(q, k, v, [[0]], [2], scale=g["scale"])
    np.testing.assert_allclose(out[0, 0], g["out"], rtol=0, atol=1e-15)


# ---------------------------------------------------------------- metadata

def test_bounds_match_numpy_min_max():
    x = _small_cache(3, 4, 2, 32, [37, 16, 70])
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    kf = x.k_cache.float().numpy().astype(np.float64)
    for b, L in enumerate(x.seq_lens.tolist()):
        for j in range(-(-L // 16)):
            phys = int(x.block_table[b, j])
            valid = min(16, L - 16 * j)
            tile = kf[phys, :, :valid, :]  # [Hkv][valid][D]
            np.testing.assert_array_equal(kmin[b, :, j], tile.min(axis=1))
            np.testing.assert_array_equal(kmax[b, :, j], tile.max(axis=1))
        assert np.isnan(kmin[b, :, -(-L // 16):]).all()


def test_bounds_ignore_slots_past_length():
    a = _small_cache(2, 2, 1, 16, [21, 40], fill="zero")
    b = _small_cache(2, 2, 1, 16, [21, 40], fill="nan")
    ka = oracle.page_bounds(a.k_cache, a.block_table, a.seq_lens)
    kb = oracle.page_bounds(b.k_cache, b.block_table, b.seq_lens)
    np.testing.assert_array_equal(ka[0], kb[0])
    np.testing.assert_array_equal(ka[1], kb[1])


# ---------------------------------------------------------------- scores

def _group_dots(x, b, h, j):
    """q_h' . k_t for every query head h' of kv head h and token t of page j."""
    G = x.q.shape[1] // x.k_cache.shape[1]
    L = int(x.seq_lens[b])
    phys = int(x.block_table[b, j])
    valid = min(16, L - 16 * j)
    k = x.k_cache[phys, h, :valid].double().numpy()
    q = x.q[b, h * G:(h + 1) * G].double().numpy()
    return q @ k.T  # [G][valid]


def test_score_is_upper_bound_on_group_logits():
    x = _small_cache(2, 8, 2, 64, [400, 333], seed=11)
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    s = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, prefix=16, window=48)
    checked = 0
    for b, L in enumerate(x.seq_lens.tolist()):
        n, npre, ws = oracle.page_ranges(L, 16, 48)
        for h in range(2):
            for j in range(npre, ws):
                dots = _group_dots(x, b, h, j)
                # the bound holds per head, hence for the group sum of the
                # per-token logits and for the largest single-head logit
                assert s[b, h, j] >= dots.sum(axis=0).max() - 1e-9
                per_head = dots.max(axis=1).sum()
                assert s[b, h, j] >= per_head - 1e-9
                checked += 1
            outside = [j for j in range(s.shape[2]) if not npre <= j < ws]
            assert np.isnan(s[b, h, outside]).all()
    assert checked > 20


def test_score_exact_when_page_tokens_equal():
    x = _small_cache(1, 4, 1, 32, [64], seed=3)
    x.k_cache[int(x.block_table[0, 2]), 0, :, :] = x.k_cache[int(x.block_table[0, 2]), 0, 5, :]
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    s = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, prefix=0, window=0)
    dots = _group_dots(x, 0, 0, 2)
    assert s[0, 0, 2] == pytest.approx(dots[:, 0].sum(), rel=1e-14, abs=1e-12)


def test_score_nonnegative_query_uses_kmax():
    x = _small_cache(1, 4, 2, 32, [160], seed=4)
    x.q.copy_(x.q.abs())
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    s = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, prefix=0, window=0)
    q = x.q.double().numpy()
    for h in range(2):
        want = kmax[0, h, :10] @ q[0, 2 * h:2 * h + 2].sum(axis=0)
        np.testing.assert_allclose(s[0, h, :10], want, rtol=1e-13)
    x.q.copy_(-x.q)
    s = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, prefix=0, window=0)
    q = x.q.double().numpy()
    for h in range(2):
        want = kmin[0, h, :10] @ q[0, 2 * h:2 * h + 2].sum(axis=0)
        np.testing.assert_allclose(s[0, h, :10], want, rtol=1e-13)


def test_score_equals_the_sign_split_form():
    """For a <= b, max(q*a, q*b) is q*b when q >= 0 and q*a otherwise, so the
    group score is also sum_d Qneg_d * kmin_d + Qpos_d * kmax_d with Qpos_d =
    sum_h max(q_hd, 0), Qneg_d = sum_h min(q_hd, 0) (the form the GPU scoring
    evaluates).  Mixed-sign queries and bounds, zeros, group sizes 1 to 8."""
    for hq, hkv, seed in [(8, 8, 21), (8, 2, 22), (12, 4, 23), (8, 1, 24)]:
        x = _small_cache(2, hq, hkv, 64, [700, 513], seed=seed)
        x.q[0, 0, :8] = 0.0
        kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
        s = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, prefix=16, window=64)
        q = x.q.double().numpy()
        G = hq // hkv
        for b, L in enumerate(x.seq_lens.tolist()):
            n, npre, ws = oracle.page_ranges(L, 16, 64)
            for h in range(hkv):
                qg = q[b, h * G:(h + 1) * G]
                qpos = np.maximum(qg, 0.0).sum(axis=0)
                qneg = np.minimum(qg, 0.0).sum(axis=0)
                want = kmin[b, h, npre:ws] @ qneg + kmax[b, h, npre:ws] @ qpos
                np.testing.assert_allclose(s[b, h, npre:ws], want, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- selection

def _brute_force_select(vals, pages, k):
    """Max-sum k-subset; ties resolved to the lexicographically smallest
    ascending page tuple.  vals are integers, so sums are exact."""
    best = None
    for combo in itertools.combinations(range(len(pages)), k):
        key = (sum(vals[i] for i in combo), [-pages[i] for i in combo])
        if best is None or key > best[0]:
            best = (key, [pages[i] for i in combo])
    return sorted(best[1]) if best else []


def test_select_matches_brute_force():
    rng = np.random.default_rng(7)
    for trial in range(60):
        npre = int(rng.integers(0, 3))
        ncand = int(rng.integers(1, 12))
        nwin = int(rng.integers(1, 3))
        n = npre + ncand + nwin
        L = 16 * n - int(rng.integers(0, 15))
        P = 16 * npre
        W = L - 16 * (npre + ncand)
        assert oracle.page_ranges(L, P, W) == (n, npre, npre + ncand)
        vals = rng.integers(-3, 4, size=ncand).tolist()  # many ties
        scores = np.full((1, 1, n), np.nan)
        scores[0, 0, npre:npre + ncand] = vals
        pages = list(range(npre, npre + ncand))
        for k in range(0, ncand + 2):
            sel, nsel = oracle.select_pages(scores, [L], P, W, k)
            got = [int(p) for p in sel[0, 0] if p >= 0]
            assert got == _brute_force_select(vals, pages, min(k, ncand)), (trial, k)


# ---------------------------------------------------------------- attention

def _sdpa(q, k, v, scale):
    """torch scaled_dot_product_attention in fp64 for one query vector."""
    return torch.nn.functional.scaled_dot_product_attention(
        q[None, None, None, :], k[None, None], v[None, None], scale=scale)[0, 0, 0]


def _gather(x, b, h, tokens):
    idx = torch.tensor(tokens, dtype=torch.long)
    phys = x.block_table[b].long()[idx // 16]
    k = x.k_cache[phys, h, idx % 16].double()
    v = x.v_cache[phys, h, idx % 16].double()
    return k, v


def test_dense_matches_torch_sdpa():
    x = _small_cache(3, 6, 2, 48, [1, 45, 130], seed=21, fill="nan")
    out = oracle.dense_decode(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens)
    scale = 1 / math.sqrt(48)
    for b, L in enumerate(x.seq_lens.tolist()):
        for hh in range(6):
            k, v = _gather(x, b, hh // 3, list(range(L)))
            want = _sdpa(x.q[b, hh].double(), k, v, scale)
            np.testing.assert_allclose(out[b, hh], want.numpy(), rtol=0, atol=1e-13)


def test_empty_sequence_gives_zero():
    x = _small_cache(2, 2, 1, 16, [0, 20], seed=2)
    out = oracle.dense_decode(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens)
    assert (out[0] == 0).all() and np.isfinite(out[1]).all()


def test_uniform_values_give_uniform_output():
    x = _small_cache(2, 4, 2, 32, [77, 300], seed=8)
    x.v_cache.fill_(1.0)
    out, _, _ = oracle.sparse_decode(x.q, x.k_cache, x.v_cache, x.block_table,
                                     x.seq_lens, prefix=16, window=32, budget=3)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_full_coverage_equals_dense():
    x = _small_cache(2, 8, 2, 64, [500, 260], seed=9)
    dense = oracle.dense_decode(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens)
    for P, W in [(16, 48), (0, 1), (64, 0)]:
        out, sel, nsel = oracle.sparse_decode(x.q, x.k_cache, x.v_cache, x.block_table,
                                              x.seq_lens, prefix=P, window=W, budget=64)
        np.testing.assert_allclose(out, dense, rtol=0, atol=1e-14)


def test_budget_zero_is_prefix_plus_window():
    x = _small_cache(2, 4, 2, 32, [333, 90], seed=12)
    P, W = 20, 50
    out, sel, nsel = oracle.sparse_decode(x.q, x.k_cache, x.v_cache, x.block_table,
                                          x.seq_lens, prefix=P, window=W, budget=0)
    assert (nsel == 0).all()
    for b, L in enumerate(x.seq_lens.tolist()):
        lo = 16 * (-(-P // 16))  # end of the last page touching [0, P)
        hi = 16 * ((L - W) // 16)  # start of the first page touching [L-W, L)
        tokens = [t for t in range(L) if t < lo or t >= hi]
        for hh in range(4):
            k, v = _gather(x, b, hh // 2, tokens)
            want = _sdpa(x.q[b, hh].double(), k, v, 1 / math.sqrt(32))
            np.testing.assert_allclose(out[b, hh], want.numpy(), rtol=0, atol=1e-13)


def test_selected_pages_attended_exactly():
    x = _small_cache(1, 4, 1, 32, [400], seed=13)
    P, W, K = 16, 32, 4
    out, sel, nsel = oracle.sparse_decode(x.q, x.k_cache, x.v_cache, x.block_table,
                                          x.seq_lens, prefix=P, window=W, budget=K)
    pages = sorted(set([0] + list(range(23, 25)) + sel[0, 0].tolist()))
    tokens = [t for t in range(400) if t // 16 in pages]
    for hh in range(4):
        k, v = _gather(x, 0, 0, tokens)
        want = _sdpa(x.q[0, hh].double(), k, v, 1 / math.sqrt(32))
        np.testing.assert_allclose(out[0, hh], want.numpy(), rtol=0, atol=1e-13)


def test_layout_invariance():
    a = _small_cache(3, 4, 2, 32, [100, 257, 31], layout="contiguous", seed=14)
    b = _small_cache(3, 4, 2, 32, [100, 257, 31], layout="shuffled", seed=14)
    assert not torch.equal(a.block_table, b.block_table)
    ra = oracle.sparse_decode(a.q, a.k_cache, a.v_cache, a.block_table, a.seq_lens, 16, 32, 2)
    rb = oracle.sparse_decode(b.q, b.k_cache, b.v_cache, b.block_table, b.seq_lens, 16, 32, 2)
    for u, w in zip(ra, rb):
        np.testing.assert_array_equal(u, w)


def test_units_are_independent():
    # one (sequence, kv head) unit alone -- its pages, its query group, one
    # kv head -- gives that unit's slice of the whole step (the selection is
    # per unit), which is what the threaded CPU baseline relies on
    x = _small_cache(3, 8, 2, 32, [300, 190, 77], layout="shuffled", seed=16)
    P, W, K = 16, 48, 3
    G = 4
    out, sel, nsel = oracle.sparse_decode(x.q, x.k_cache, x.v_cache, x.block_table,
                                          x.seq_lens, P, W, K)
    for b, L in enumerate(x.seq_lens.tolist()):
        n = -(-L // 16)
        phys = x.block_table[b, :n].long()
        for h in range(2):
            o, s_, ns = oracle.sparse_decode(
                x.q[b:b + 1, h * G:(h + 1) * G].contiguous(),
                x.k_cache[phys, h:h + 1].contiguous(), x.v_cache[phys, h:h + 1].contiguous(),
                torch.arange(n, dtype=torch.int32).reshape(1, n), x.seq_lens[b:b + 1], P, W, K)
            np.testing.assert_array_equal(o[0], out[b, h * G:(h + 1) * G])
            np.testing.assert_array_equal(s_[0, 0], sel[b, h])
            assert ns[0, 0] == nsel[b, h]


def test_composition_of_steps():
    x = _small_cache(2, 4, 2, 32, [300, 190], seed=15)
    P, W, K = 32, 40, 3
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    s = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, P, W)
    sel, nsel = oracle.select_pages(s, x.seq_lens, P, W, K)
    out = oracle.attend(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, P, W, sel)
    out2, sel2, nsel2 = oracle.sparse_decode(x.q, x.k_cache, x.v_cache, x.block_table,
                                             x.seq_lens, P, W, K)
    np.testing.assert_array_equal(sel, sel2)
    np.testing.assert_array_equal(out, out2)


def test_needles_are_selected_tiny_workload():
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(wl)
    out, sel, nsel = oracle.sparse_decode(x.q, x.k_cache, x.v_cache, x.block_table,
                                          x.seq_lens, x.prefix, x.window, x.budget)
    assert len(x.needle_tokens[0]) == wl.needles
    for h in range(wl.hkv):
        chosen = set(sel[0, h].tolist())
        for t in x.needle_tokens[0]:
            assert t // 16 in chosen


# ---------------------------------------------------------------- fp8 metadata

def test_fp8_rounding_golden():
    """Hand-worked E4M3 outward roundings (tests/golden/fp8_rounding.json)."""
    for c in _load("fp8_rounding.json")["cases"]:
        assert oracle.fp8_round(c["x"], True) == c["up"], c
        assert oracle.fp8_round(c["x"], False) == c["down"], c


def _e4m3_table():
    """Every finite E4M3 value, from torch's float8_e4m3fn dtype (a library
    definition of the format, independent of the oracle)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return codes.numpy(), vals


def test_fp8_values_match_library_format():
    codes, vals = _e4m3_table()
    for c, v in zip(codes, vals):
        if np.isnan(v):  # the two NaN codes: the out-of-range bounds
            assert abs(oracle.fp8_value(int(c))) == 3.3895313892515355e38
            assert (oracle.fp8_value(int(c)) > 0) == (c == 0x7F)
        else:
            assert oracle.fp8_value(int(c)) == v, c


def test_fp8_rounding_is_outward_and_tight():
    """For bf16 values over the whole range (tiny, subnormal in E4M3, normal,
    beyond 448): down <= x <= up, and no E4M3 value lies strictly between x
    and either (checked against the library's value table)."""
    _, vals = _e4m3_table()
    finite = np.unique(vals[~np.isnan(vals)])
    g = torch.Generator().manual_seed(7)
    xs = torch.cat([torch.randn(3000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 600.0)])
    xs = xs.to(torch.bfloat16).double().numpy()
    for x in xs:
        up, dn = oracle.fp8_round(x, True), oracle.fp8_round(x, False)
        vu, vd = oracle.fp8_value(up), oracle.fp8_value(dn)
        assert vd <= x <= vu, (x, vd, vu)
        assert not ((finite > x) & (finite < vu)).any(), x
        assert not ((finite < x) & (finite > vd)).any(), x


def test_fp8_page_bounds_round_the_exact_bounds_outward():
    """E4M3 page bounds are the exact bounds rounded outward, and the score
    from them bounds the score from the exact bounds, which bounds every
    group logit of the page (fp64)."""
    x = _small_cache(2, 8, 2, 64, [400, 333], seed=13)
    x.k_cache = (x.k_cache.float() * 3).to(torch.bfloat16)  # some keys beyond +-1
    kmin, kmax = oracle.page_bounds(x.k_cache, x.block_table, x.seq_lens)
    c8min, c8max = oracle.page_bounds_fp8(x.k_cache, x.block_table, x.seq_lens)
    m8, M8 = oracle.fp8_decode(c8min), oracle.fp8_decode(c8max)
    for b, L in enumerate(x.seq_lens.tolist()):
        n = -(-L // 16)
        assert (m8[b, :, :n] <= kmin[b, :, :n]).all()
        assert (M8[b, :, :n] >= kmax[b, :, :n]).all()
        for h in range(2):
            for j in range(n):
                for d in range(0, 64, 7):
                    assert c8min[b, h, j, d] == oracle.fp8_round(kmin[b, h, j, d], False)
                    assert c8max[b, h, j, d] == oracle.fp8_round(kmax[b, h, j, d], True)
    s = oracle.page_scores(x.q, kmin, kmax, x.seq_lens, prefix=16, window=48)
    s8 = oracle.page_scores(x.q, m8, M8, x.seq_lens, prefix=16, window=48)
    cand = ~np.isnan(s)
    assert (s8[cand] >= s[cand]).all()
    for b in range(2):
        for h in range(2):
            for j in np.nonzero(cand[b, h])[0][::5]:
                assert s8[b, h, j] >= _group_dots(x, b, h, j).sum(axis=0).max() - 1e-9


def test_fp8_bounds_of_a_page_grow_one_token_at_a_time():
    """Outward rounding is monotone, so the bounds of a page with one more
    token are the old codes combined with the new token's rounded values
    (min of the downs, max of the ups): appending keeps fp8 metadata exact."""
    x = _small_cache(1, 4, 2, 32, [16], seed=17)
    bt = x.block_table
    for t in range(1, 16):
        a8 = oracle.page_bounds_fp8(x.k_cache, bt, [t])
        b8 = oracle.page_bounds_fp8(x.k_cache, bt, [t + 1])
        k = x.k_cache[int(bt[0, 0]), :, t].double().numpy()  # [Hkv][D]
        for h in range(2):
            for d in range(32):
                dn = oracle.fp8_round(k[h, d], False)
                up = oracle.fp8_round(k[h, d], True)
                lo = min(oracle.fp8_value(a8[0][0, h, 0, d]), oracle.fp8_value(dn))
                hi = max(oracle.fp8_value(a8[1][0, h, 0, d]), oracle.fp8_value(up))
                assert oracle.fp8_value(b8[0][0, h, 0, d]) == lo
                assert oracle.fp8_value(b8[1][0, h, 0, d]) == hi


# ------------------------------------------------------------------ top-delta

def _delta_scores(fx):
    n = -(-fx["length"] // 16)
    s = np.full((1, 1, n), np.nan)
    s[0, 0, :] = fx["scores"]
    return s


def test_top_delta_golden():
    fx = json.load(open(os.path.join(GOLDEN, "top_delta.json")))
    s = _delta_scores(fx)
    for c in fx["cases"]:
        sel, nsel = oracle.select_pages_delta(s, [fx["length"]], fx["prefix"], fx["window"],
                                              c["d"], c["delta"], c["cap"])
        want = c["selected"] + [-1] * (c["cap"] - len(c["selected"]))
        assert sel[0, 0].tolist() == want, c
        assert int(nsel[0, 0]) == len(c["selected"]), c


def test_top_delta_is_a_longer_top_k():
    """The top d and the pages within delta of the best are both prefixes of
    the (score desc, page asc) order, so their union is the top k with
    k = max(d, #within delta), capped: the plain selection with that budget."""
    rng = np.random.default_rng(5)
    for trial in range(40):
        B, hkv, mp = 2, 2, 90
        lens = rng.integers(1, mp * 16, size=B).astype(np.int32)
        prefix, window = int(rng.integers(0, 60)), int(rng.integers(0, 300))
        s = np.round(rng.normal(size=(B, hkv, mp)) * 4) / 4  # many exact ties
        d = int(rng.integers(0, 12))
        delta = float(rng.choice([0.0, 0.25, 0.5, 1.0, 2.5]))
        cap = int(rng.integers(1, 40))
        sel, nsel = oracle.select_pages_delta(s, lens, prefix, window, d, delta, cap)
        for b in range(B):
            n, np_, ws = oracle.page_ranges(int(lens[b]), prefix, window)
            for h in range(hkv):
                cand = s[b, h, np_:ws]
                m = int((cand.max() - cand <= delta).sum()) if cand.size else 0
                k = min(max(d, m), cap, cand.size)
                ref, rn = oracle.select_pages(s[b:b + 1, h:h + 1], lens[b:b + 1], prefix, window, k)
                assert int(nsel[b, h]) == k == int(rn[0, 0])
                assert sel[b, h, :k].tolist() == ref[0, 0, :k].tolist()
                assert (sel[b, h, k:] == -1).all()


def test_top_delta_edges():
    rng = np.random.default_rng(6)
    s = rng.normal(size=(1, 2, 50))
    lens = [800]
    top, _ = oracle.select_pages(s, lens, 16, 64, 7)
    neg, nn = oracle.select_pages_delta(s, lens, 16, 64, 7, -1.0, 7)
    assert (neg == top).all() and (nn == 7).all()  # a negative delta adds nothing
    n, np_, ws = oracle.page_ranges(800, 16, 64)
    allc, na = oracle.select_pages_delta(s, lens, 16, 64, 0, np.inf, 60)
    assert (na == ws - np_).all()  # an infinite delta keeps every candidate
    assert allc[0, 0, : ws - np_].tolist() == list(range(np_, ws))
