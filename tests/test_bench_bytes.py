"""The benchmark's byte accounting (CPU): bench.py's page ranges agree with
the oracle's, and its algorithmic bytes equal the bytes of the pages and
tokens the oracle actually reads and attends."""
import itertools

import numpy as np

import bench
import oracle
import synth


def test_page_ranges_match_oracle():
    for L, P, W in itertools.product([0, 1, 15, 16, 17, 100, 255, 256, 257, 4096],
                                     [0, 1, 16, 17, 64, 300],
                                     [0, 1, 16, 17, 256, 5000]):
        assert bench.page_ranges(L, P, W) == oracle.page_ranges(L, P, W), (L, P, W)


def _count(x, prefix, window, budget):
    """Metadata and K/V bytes the oracle's step reads, counted from its own
    page ranges and selection."""
    _, sel, nsel = oracle.sparse_decode(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens,
                                        prefix, window, budget)
    hkv, D = x.k_cache.shape[1], x.k_cache.shape[3]
    meta = forced = chosen = 0
    for b, L in enumerate(x.seq_lens.tolist()):
        n, np_, ws = oracle.page_ranges(L, prefix, window)
        meta += (ws - np_) * hkv * 4 * D
        for h in range(hkv):
            fpages = set(range(np_)) | set(range(ws, n))
            spages = set(int(p) for p in sel[b, h, :int(nsel[b, h])]) - fpages
            forced += sum(min(16, L - 16 * j) for j in fpages) * 4 * D
            chosen += sum(min(16, L - 16 * j) for j in spages) * 4 * D
    return meta, forced, chosen


def test_algorithmic_bytes_equal_what_the_oracle_reads():
    wl = synth.Workload(name="t", batch=3, hq=8, hkv=2, head_dim=32, prefix=40, window=100,
                        budget=5, needles=0, seed=11, context=1000, layout="shuffled")
    x = synth.make_inputs(wl, lens_override=[1000, 333, 130])
    for prefix, window, budget in [(40, 100, 5), (0, 16, 3), (64, 256, 50), (16, 17, 0)]:
        meta, forced, chosen = _count(x, prefix, window, budget)
        total, m, k = bench.algorithmic_bytes(x.seq_lens.tolist(), 8, 2, 32, prefix, window,
                                               budget)
        assert (m, k) == (meta, forced + chosen), (prefix, window, budget)
        assert total == meta + forced + chosen + 3 * 8 * 32 * (2 + 4)  # q bf16 + out fp32
        st = bench.stage_bytes(x.seq_lens.tolist(), 8, 2, 32, prefix, window, budget)
        assert st[1] == meta + forced + 3 * 8 * 32 * 2  # streaming kernel: + q
        assert st[2] == chosen + 3 * 8 * 32 * (2 + 4)  # finishing kernel: + q, out
        assert st[1] + st[2] == total + 3 * 8 * 32 * 2  # q is read by both


def test_dense_bytes_are_every_token():
    lens = [1000, 333, 130]
    total, m, k = bench.algorithmic_bytes(lens, 8, 2, 32, 0, 0, 0, dense=True)
    assert m == 0
    assert k == sum(lens) * 2 * 4 * 32
    assert np.isclose(total, k + 3 * 8 * 32 * 6)


def test_e4m3_metadata_halves_the_metadata_bytes():
    lens = [1000, 333, 130]
    t2, m2, k2 = bench.algorithmic_bytes(lens, 8, 2, 32, 40, 100, 5)
    t1, m1, k1 = bench.algorithmic_bytes(lens, 8, 2, 32, 40, 100, 5, meta_bytes=1)
    assert m1 * 2 == m2 and k1 == k2 and t2 - t1 == m1
