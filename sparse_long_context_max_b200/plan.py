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
graph.  The per-step inputs live in one device byte buffer, so a caller
feeding them from the host moves them with a single copy (``host_buffers``,
``run_from_host``).  This module orders calls only: every step of the path
runs in the library's kernels.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch

from . import (PagedCache, dense_decode, kv_append, sparse_attend, sparse_decode,
               workspace_size)

__all__ = ["LayerSpec", "index_reuse", "DecodeStep", "StepIO", "packed_layout"]

_ALIGN = 256  # byte alignment of every tensor inside the packed input buffer


def packed_layout(num_layers: int, batch: int, num_q_heads: int, num_kv_heads: int,
                  head_dim: int):
    """Byte layout of a step's inputs in one buffer: (name, offset, shape,
    dtype) for q (bf16 [layers][B][Hq][D]), k_new and v_new (bf16
    [layers][B][Hkv][D]), positions and seq_lens (int32 [B]), each at an
    offset that is a multiple of 256 bytes; and the total size."""
    items = [("q", (num_layers, batch, num_q_heads, head_dim), torch.bfloat16),
             ("k_new", (num_layers, batch, num_kv_heads, head_dim), torch.bfloat16),
             ("v_new", (num_layers, batch, num_kv_heads, head_dim), torch.bfloat16),
             ("positions", (batch,), torch.int32),
             ("seq_lens", (batch,), torch.int32)]
    out, off = [], 0
    for name, shape, dt in items:
        n = 1
        for v in shape:
            n *= v
        out.append((name, off, shape, dt))
        off += -(-n * torch.empty((), dtype=dt).element_size() // _ALIGN) * _ALIGN
    return out, off


def _views(buf: torch.Tensor, layout) -> dict:
    views = {}
    for name, off, shape, dt in layout:
        n = 1
        for v in shape:
            n *= v
        nb = n * torch.empty((), dtype=dt).element_size()
        views[name] = buf[off:off + nb].view(dt).view(shape)
    return views


@dataclasses.dataclass
class StepIO:
    """Pinned host buffers mirroring a DecodeStep's inputs and outputs.

    inputs     uint8, the packed bytes (copied to the device in one copy)
    q, k_new, v_new, positions, seq_lens   views into ``inputs``
    out        fp32 [layers][B][Hq][D], filled by ``run_from_host``
    """

    inputs: torch.Tensor
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    positions: torch.Tensor
    seq_lens: torch.Tensor
    out: torch.Tensor


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
        self.layout, nbytes = packed_layout(L, B, num_q_heads, hkv, D)
        self.inputs = torch.zeros((nbytes,), dtype=torch.uint8, device=dev)
        v = _views(self.inputs, self.layout)
        self.q, self.k_new, self.v_new = v["q"], v["k_new"], v["v_new"]
        self.positions, self.seq_lens = v["positions"], v["seq_lens"]
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

    def host_buffers(self) -> StepIO:
        """Pinned host buffers laid out like this step's inputs and output."""
        buf = torch.zeros(self.inputs.shape, dtype=torch.uint8).pin_memory()
        v = _views(buf, self.layout)
        out = torch.zeros(self.out.shape, dtype=torch.float32).pin_memory()
        return StepIO(buf, v["q"], v["k_new"], v["v_new"], v["positions"], v["seq_lens"], out)

    def run_from_host(self, io: StepIO):
        """Issue, on the current stream: one host-to-device copy of
        ``io.inputs``, the step (its graph), one device-to-host copy of the
        outputs into ``io.out``.  Asynchronous: synchronise before reading
        ``io.out`` or rewriting ``io.inputs``."""
        self.inputs.copy_(io.inputs, non_blocking=True)
        self.replay()
        io.out.copy_(self.out, non_blocking=True)
