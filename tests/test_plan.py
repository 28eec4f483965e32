"""Host logic of the multi-layer decode step (CPU only): the Full/Shared
assignment of cross-layer reuse and the packed input layout that lets a
caller move a step's inputs with one copy."""
import pytest
import torch

from sparse_long_context_max_b200 import plan as P


def test_index_reuse_keeps_every_fourth_sparse_layer():
    specs = [P.LayerSpec(512, 64), P.LayerSpec(0, 0, dense=True)] + \
        [P.LayerSpec(256 * (i + 1), 32) for i in range(9)]
    got = P.index_reuse(specs, every=4)
    sparse = [s for s in got if not s.dense]
    assert [s.shared for s in sparse] == [(k % 4) != 0 for k in range(len(sparse))]
    assert got[1].dense and not got[1].shared
    assert [(s.window, s.budget) for s in got] == [(s.window, s.budget) for s in specs]
    assert all(not s.shared for s in P.index_reuse(specs, every=1))


def test_packed_layout_is_aligned_and_disjoint():
    for L, B, hq, hkv, D in [(1, 1, 8, 2, 128), (15, 4, 16, 2, 256), (3, 7, 12, 3, 128)]:
        layout, total = P.packed_layout(L, B, hq, hkv, D)
        names = [n for n, _, _, _ in layout]
        assert names == ["q", "k_new", "v_new", "positions", "seq_lens"]
        spans = []
        for name, off, shape, dt in layout:
            assert off % 256 == 0
            n = 1
            for v in shape:
                n *= v
            spans.append((off, off + n * torch.empty((), dtype=dt).element_size()))
        spans.sort()
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
        assert spans[-1][1] <= total and total % 256 == 0
        assert dict((n, s) for n, _, s, _ in layout)["q"] == (L, B, hq, D)
        assert dict((n, s) for n, _, s, _ in layout)["k_new"] == (L, B, hkv, D)


def test_packed_views_round_trip_through_one_copy():
    """Values written through one buffer's views arrive, after a single byte
    copy, in the other buffer's views."""
    layout, total = P.packed_layout(2, 3, 8, 2, 128)
    src = torch.zeros(total, dtype=torch.uint8)
    dst = torch.zeros(total, dtype=torch.uint8)
    vs, vd = P._views(src, layout), P._views(dst, layout)
    g = torch.Generator().manual_seed(3)
    want = {}
    for name, t in vs.items():
        if t.dtype == torch.int32:
            t.copy_(torch.randint(0, 1 << 20, t.shape, generator=g, dtype=torch.int32))
        else:
            t.copy_(torch.randn(t.shape, generator=g).to(t.dtype))
        want[name] = t.clone()
    dst.copy_(src)
    for name, t in vd.items():
        assert torch.equal(t, want[name]), name


class _CacheShape:
    """Stands in for a PagedCache: DecodeStep reads only its shape before
    it checks the plan."""
    num_kv_heads, head_dim = 2, 128


def test_decode_step_rejects_a_bad_plan():
    bt = torch.zeros((2, 8), dtype=torch.int32)
    caches = [_CacheShape(), _CacheShape()]
    with pytest.raises(ValueError):  # a Shared layer needs a Full layer before it
        P.DecodeStep(caches, bt, [P.LayerSpec(256, 16, shared=True), P.LayerSpec(256, 16)],
                     prefix=16, num_q_heads=8)
    with pytest.raises(ValueError):  # one cache per layer
        P.DecodeStep(caches[:1], bt, [P.LayerSpec(256, 16), P.LayerSpec(256, 16)],
                     prefix=16, num_q_heads=8)
