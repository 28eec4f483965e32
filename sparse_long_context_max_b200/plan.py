"""One decode step over a stack of full-attention layers.

A hybrid model's remaining full-attention layers each get their own sliding
window and selection budget, and some stay dense ("Hybrid LLM Decoding 2.2x
Faster at 256k, No Retraining", sections "The method: sliding window +
prefix + query-aware pages, searched per layer" and "Why it matters").
Cross-layer index reuse ("IndexCache: cross-layer reuse speeds 30B prefill
1.82x") adds a second kind of sparse layer: a Full layer selects its pages;
a Shared layer skips scoring and selection and attends the selection of the
nearest Full layer before it, together with its own prefix and window.

``DecodeStep`` owns the static device buffers of one step (the new token's
q, k and v per layer, the positions, the lengths, the outputs and the Full
layers' selections) and runs, per layer, ``kv_append`` then that layer's
decode through the C ABI; ``capture()`` records the whole step as one CUDA
graph.  This module orders calls only: every step of the path runs in the
library's kernels.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch

from . import (PagedCache, dense_decode, kv_append, sparse_attend, sparse_decode,
               workspace_size)

__all__ = ["LayerSpec", "index_reuse", "DecodeStep"]


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """One full-attention layer of the step.

    window, budget  sliding window (tokens) and selection budget (pages)
    dense           attend every token (no prefix/window/selection)
    shared          reuse the selection of the nearest preceding Full layer
                    (a sparse layer that is not shared) instead of selecting
    """

    window: int
    budget: int
    dense: bool = False
    shared: bool = False


def index_reuse(specs: Sequence[LayerSpec], every: int = 4) -> List[LayerSpec]:
    """The plan with cross-layer selection reuse: among the sparse layers,
    in order, the first and then every ``every``-th selects its pages (Full)
    and the others reuse the nearest Full layer's selection (Shared).  With
    every = 4 a quarter of the sparse layers keep their selection, matching
    the 75% cut in indexer work IndexCache reports."""
    out, k = [], 0
    for s in specs:
        if s.dense:
            out.append(dataclasses.replace(s, shared=False))
            continue
        out.append(dataclasses.replace(s, shared=(k % every) != 0))
        k += 1
    return out


class DecodeStep:
    """Static buffers and the launch sequence of one decode step.

    caches       one PagedCache per layer (same page pool shape)
    block_table  int32 [B][max_pages] (shared by the layers)
    specs        one LayerSpec per layer
    prefix       pinned prefix (tokens), shared by the sparse layers
    num_q_heads  query heads per layer

    Fill ``q[i]``, ``k_new[i]``, ``v_new[i]`` (layer i's new token),
    ``positions`` (each sequence's slot for the new token, i.e. its length
    before the step) and ``seq_lens`` (``positions + 1``: the new token
    attends to itself), then call ``run()`` or ``replay()``.  Results:
    ``out[i]`` (fp32 [B][Hq][D]) and, for Full layers, ``selected[i]``
    (int32 [B][Hkv][budget]).
    """

    def __init__(self, caches: Sequence[PagedCache], block_table: torch.Tensor,
                 specs: Sequence[LayerSpec], prefix: int, num_q_heads: int):
        if len(caches) != len(specs):
            raise ValueError("one cache per layer")
        self.caches = list(caches)
        self.specs = list(specs)
        self.bt = block_table
        self.prefix = prefix
        dev = block_table.device
        B, mp = block_table.shape
        hkv, D = caches[0].num_kv_heads, caches[0].head_dim
        self.full_of: List[Optional[int]] = []
        last_full = None
        for i, s in enumerate(self.specs):
            if s.dense:
                self.full_of.append(None)
            elif s.shared:
                if last_full is None:
                    raise ValueError("layer %d is Shared but no Full layer precedes it" % i)
                self.full_of.append(last_full)
            else:
                last_full = i
                self.full_of.append(i)
        L = len(self.specs)
        self.q = torch.zeros((L, B, num_q_heads, D), dtype=torch.bfloat16, device=dev)
        self.k_new = torch.zeros((L, B, hkv, D), dtype=torch.bfloat16, device=dev)
        self.v_new = torch.zeros((L, B, hkv, D), dtype=torch.bfloat16, device=dev)
        self.positions = torch.zeros((B,), dtype=torch.int32, device=dev)
        self.seq_lens = torch.zeros((B,), dtype=torch.int32, device=dev)
        self.out = torch.zeros((L, B, num_q_heads, D), dtype=torch.float32, device=dev)
        self.selected = {i: torch.full((B, hkv, max(s.budget, 1)), -1, dtype=torch.int32,
                                       device=dev)[:, :, : s.budget].contiguous()
                         for i, s in enumerate(self.specs) if not s.dense and not s.shared}
        kmax = max([s.budget for s in self.specs if not s.dense] + [0])
        self.workspace = torch.empty(workspace_size(B, num_q_heads, hkv, D, mp, kmax),
                                     dtype=torch.uint8, device=dev)
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    def launches(self) -> int:
        """Kernels one step launches: per layer, the append and the two
        kernels of its decode."""
        return 3 * len(self.specs)

    def run(self):
        """Issue the step on the current stream."""
        for i, s in enumerate(self.specs):
            c = self.caches[i]
            kv_append(c, self.k_new[i], self.v_new[i], self.bt, self.positions)
            if s.dense:
                dense_decode(self.q[i], c, self.bt, self.seq_lens, out=self.out[i],
                             workspace=self.workspace)
            elif s.shared:
                sparse_attend(self.q[i], c, self.bt, self.seq_lens, self.prefix, s.window,
                              self.selected[self.full_of[i]], out=self.out[i],
                              workspace=self.workspace)
            else:
                sparse_decode(self.q[i], c, self.bt, self.seq_lens, self.prefix, s.window,
                              s.budget, out=self.out[i], selected_out=self.selected[i],
                              workspace=self.workspace)

    def capture(self) -> torch.cuda.CUDAGraph:
        """Run the step once (the library's per-device set-up happens
        outside the capture), then record it as one CUDA graph."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run()
        torch.cuda.synchronize()
        self.graph = g
        return g

    def replay(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()
