"""Seeded synthetic inputs for decode-step combined sparse attention.

This module draws inputs only: queries, a paged bf16 K/V cache, planted
"needle" keys, sequence lengths, block tables and per-step appended tokens.
It contains none of the method's arithmetic (no metadata, scores, selection
or attention), so both the CUDA path and the CPU oracle can consume it.

Every tensor is produced on the host by ``torch`` CPU generators, in
independently seeded chunks (one chunk = a run of logical pages of one
sequence), so the values are the same whatever the physical page layout and
whatever the number of worker threads.  Values are drawn as fp32 N(0, 1) and
rounded to bf16 (round-to-nearest-even, torch's conversion).

The workloads mirror the shapes of the long-context decode runs described in
"Hybrid LLM Decoding 2.2x Faster at 256k, No Retraining" (section "Results
and limits: a free 2x, and where you don't get it": 64k and 256k context at
batch 4; section "Why it matters": 15 full-attention layers with per-layer
windows from 256 to 4096, two of them left dense).  The pages' own runs use
real models and long-context datasets; these synthetic tensors stand in for
them.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import torch

PAGE = 16  # tokens per KV page

__all__ = [
    "PAGE",
    "Workload",
    "WORKLOADS",
    "Inputs",
    "make_inputs",
    "step_tokens",
    "layer_query",
    "layer_plan",
    "chunk_seed",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic decode workload."""

    name: str
    batch: int
    hq: int
    hkv: int
    head_dim: int
    prefix: int  # pinned prefix, tokens
    window: int  # sliding window, tokens
    budget: int  # query-relevant pages kept per (sequence, kv head)
    needles: int  # planted needle keys per sequence
    seed: int
    context: int = 0  # tokens per sequence (0 => ragged draw)
    ragged_lo: int = 0
    ragged_hi: int = 0
    layout: str = "contiguous"  # or "shuffled" (shared, permuted page pool)
    steps: int = 1  # consecutive decode steps (each appends one token)
    layers: int = 1
    dense_layers: int = 0  # layers of ``layers`` that stay dense
    short: tuple = ()  # lengths that replace the first draws (ragged only)

    @property
    def group(self) -> int:
        return self.hq // self.hkv


# The five workloads.  Seeds are fixed: 1000 + index.
WORKLOADS = {
    "tiny": Workload(
        name="tiny", batch=1, context=4096, hq=8, hkv=2, head_dim=128,
        prefix=64, window=256, budget=32, needles=8, seed=1000),
    "decode64k": Workload(
        name="decode64k", batch=4, context=65536, hq=32, hkv=4, head_dim=128,
        prefix=128, window=1024, budget=128, needles=64, seed=1001, steps=256),
    "decode256k": Workload(
        name="decode256k", batch=4, context=262144, hq=32, hkv=4,
        head_dim=128, prefix=128, window=4096, budget=256, needles=64,
        seed=1002),
    "layers131k": Workload(
        name="layers131k", batch=4, context=131072, hq=16, hkv=2,
        head_dim=256, prefix=128, window=0, budget=0, needles=64, seed=1003,
        layers=15, dense_layers=2),
    "ragged": Workload(
        name="ragged", batch=32, ragged_lo=2048, ragged_hi=262144, hq=16,
        hkv=4, head_dim=128, prefix=64, window=512, budget=64, needles=8,
        seed=1004, layout="shuffled", short=(1615, 700)),
}

WINDOW_CHOICES = (256, 512, 1024, 2048, 4096)


def chunk_seed(*parts) -> int:
    """A 63-bit seed derived from the parts (stable across runs/platforms)."""
    h = hashlib.blake2b(repr(parts).encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 63) - 1)


def _randn(shape, *parts) -> torch.Tensor:
    g = torch.Generator().manual_seed(chunk_seed(*parts))
    return torch.randn(shape, generator=g, dtype=torch.float32)


def layer_plan(wl: Workload):
    """Per-layer (window, budget, dense) triples, drawn from the seed.

    window is uniform over WINDOW_CHOICES, budget uniform in [64, 512]
    pages; ``dense_layers`` layer indices (without replacement) stay dense.
    """
    if wl.layers == 1:
        return [(wl.window, wl.budget, False)]
    g = torch.Generator().manual_seed(chunk_seed(wl.seed, "layers"))
    w_idx = torch.randint(0, len(WINDOW_CHOICES), (wl.layers,), generator=g)
    budgets = torch.randint(64, 513, (wl.layers,), generator=g)
    dense = set(torch.randperm(wl.layers, generator=g)[: wl.dense_layers].tolist())
    return [(WINDOW_CHOICES[int(w_idx[i])], int(budgets[i]), i in dense)
            for i in range(wl.layers)]


def seq_lengths(wl: Workload) -> list:
    if wl.context:
        return [wl.context] * wl.batch
    g = torch.Generator().manual_seed(chunk_seed(wl.seed, "lens"))
    u = torch.rand(wl.batch, generator=g, dtype=torch.float64)
    lo, hi = math.log(wl.ragged_lo), math.log(wl.ragged_hi)
    lens = [int(math.floor(math.exp(lo + (hi - lo) * float(x)))) for x in u]
    # a log-uniform draw from 2048 tokens never yields a sequence that
    # prefix + window + budget cover whole; the first draws are replaced by
    # such short lengths (1615 tokens = exactly ``budget`` candidate pages)
    lens[: len(wl.short)] = list(wl.short)
    return lens


@dataclasses.dataclass
class Inputs:
    """One layer's decode inputs (host tensors).

    q         bf16 [B][Hq][D]
    k_cache   bf16 [num_pages][Hkv][PAGE][D]   (physical page pool)
    v_cache   bf16 [num_pages][Hkv][PAGE][D]
    block_table int32 [B][max_pages]  logical page -> physical page (-1 unused)
    seq_lens  int32 [B]
    needle_tokens  list (per sequence) of planted token positions
    """

    wl: Workload
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_table: torch.Tensor
    seq_lens: torch.Tensor
    needle_tokens: list
    prefix: int
    window: int
    budget: int
    layer: int = 0


def _fill_(t: torch.Tensor, fill: str):
    if fill == "zero":
        t.zero_()
    elif fill == "nan":
        # alternate NaN and +/-Inf sentinels so any use of them shows up
        t.fill_(float("nan"))
        flat = t.view(-1)
        flat[1::3] = float("inf")
        flat[2::3] = float("-inf")
    else:
        raise ValueError(fill)


def make_inputs(wl: Workload, layer: int = 0, fill: str = "zero",
                layout: Optional[str] = None, headroom_tokens: Optional[int] = None,
                spare_pages: int = 3, threads: int = 8,
                lens_override: Optional[list] = None,
                needles: Optional[int] = None) -> Inputs:
    """Draw one layer's inputs for ``wl``.

    ``fill`` sets the content of every cache slot that holds no token
    ("zero", or "nan" for NaN/Inf sentinels).  ``headroom_tokens`` reserves
    pages for later appends (default: the workload's step count).
    ``lens_override`` replaces the sequence lengths (same recipe otherwise).
    """
    layout = layout or wl.layout
    lens = list(lens_override) if lens_override is not None else seq_lengths(wl)
    B, Hq, Hkv, D = wl.batch, wl.hq, wl.hkv, wl.head_dim
    assert len(lens) == B
    headroom = wl.steps if headroom_tokens is None else headroom_tokens
    window, budget, _dense = layer_plan(wl)[layer]
    nalloc = [max(1, -(-(L + headroom) // PAGE)) for L in lens]
    max_pages = max(nalloc)
    total = sum(nalloc) + spare_pages
    seed = wl.seed + 7919 * layer

    # physical placement of every logical page
    bt = torch.full((B, max_pages), -1, dtype=torch.int32)
    if layout == "contiguous":
        base = 0
        for b in range(B):
            bt[b, : nalloc[b]] = torch.arange(base, base + nalloc[b], dtype=torch.int32)
            base += nalloc[b]
    elif layout == "shuffled":
        g = torch.Generator().manual_seed(chunk_seed(seed, "perm"))
        perm = torch.randperm(total, generator=g).to(torch.int32)
        base = 0
        for b in range(B):
            bt[b, : nalloc[b]] = perm[base: base + nalloc[b]]
            base += nalloc[b]
    else:
        raise ValueError(layout)

    kc = torch.empty((total, Hkv, PAGE, D), dtype=torch.bfloat16)
    vc = torch.empty((total, Hkv, PAGE, D), dtype=torch.bfloat16)
    _fill_(kc, fill)
    _fill_(vc, fill)

    q = layer_query(wl, layer)

    CH = 256  # logical pages per generator chunk
    jobs = []
    for b in range(B):
        npg = -(-lens[b] // PAGE)
        for j0 in range(0, npg, CH):
            jobs.append((b, j0, min(npg, j0 + CH)))

    def work(job):
        b, j0, j1 = job
        phys = bt[b, j0:j1].long()
        shape = (j1 - j0, Hkv, PAGE, D)
        kk = _randn(shape, seed, "k", b, j0).to(torch.bfloat16)
        vv = _randn(shape, seed, "v", b, j0).to(torch.bfloat16)
        valid_last = lens[b] - PAGE * (j1 - 1)  # tokens in the chunk's last page
        if j1 * PAGE > lens[b] and valid_last < PAGE:
            empty = 0.0 if fill == "zero" else float("nan")
            kk[-1, :, valid_last:, :] = empty
            vv[-1, :, valid_last:, :] = empty
        kc[phys] = kk
        vc[phys] = vv

    if threads > 1 and len(jobs) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, jobs))
    else:
        for job in jobs:
            work(job)

    # planted needles: at every kv head of the chosen token, the key points
    # along the mean of that kv head's query heads, with 4x the typical key
    # norm (keys are N(0,1) per dimension, so sqrt(D)); placed well clear of
    # prefix and window
    nn = wl.needles if needles is None else needles
    needle_tokens = []
    G = Hq // Hkv
    qf = q.float()
    for b in range(B):
        L = lens[b]
        lo_page = -(-(wl.prefix + PAGE) // PAGE)
        hi_page = (L - window - 2 * PAGE) // PAGE  # exclusive
        toks = []
        if nn > 0 and hi_page > lo_page:
            g = torch.Generator().manual_seed(chunk_seed(seed, "needle", b))
            npages = hi_page - lo_page
            pages = torch.randperm(npages, generator=g)[: min(nn, npages)] + lo_page
            slots = torch.randint(0, PAGE, (len(pages),), generator=g)
            for pg, sl in zip(pages.tolist(), slots.tolist()):
                toks.append(pg * PAGE + sl)
            toks.sort()
            for t in toks:
                phys = int(bt[b, t // PAGE])
                for h in range(Hkv):
                    g_mean = qf[b, h * G:(h + 1) * G, :].mean(dim=0)
                    key = 4.0 * math.sqrt(D) * g_mean / g_mean.norm()
                    kc[phys, h, t % PAGE, :] = key.to(torch.bfloat16)
        needle_tokens.append(toks)

    return Inputs(wl=wl, q=q, k_cache=kc, v_cache=vc, block_table=bt,
                  seq_lens=torch.tensor(lens, dtype=torch.int32),
                  needle_tokens=needle_tokens, prefix=wl.prefix, window=window,
                  budget=budget, layer=layer)


def layer_query(wl: Workload, layer: int = 0) -> torch.Tensor:
    """The decode query of ``layer`` (bf16 [B][Hq][D]), as make_inputs draws it."""
    seed = wl.seed + 7919 * layer
    return _randn((wl.batch, wl.hq, wl.head_dim), seed, "q", 0).to(torch.bfloat16)


def step_tokens(wl: Workload, step: int, layer: int = 0):
    """Fresh (q, k_new, v_new) for decode step ``step`` (step >= 1).

    q bf16 [B][Hq][D]; k_new, v_new bf16 [B][Hkv][D].
    """
    seed = wl.seed + 7919 * layer
    B, Hq, Hkv, D = wl.batch, wl.hq, wl.hkv, wl.head_dim
    q = _randn((B, Hq, D), seed, "q", step).to(torch.bfloat16)
    kn = _randn((B, Hkv, D), seed, "knew", step).to(torch.bfloat16)
    vn = _randn((B, Hkv, D), seed, "vnew", step).to(torch.bfloat16)
    return q, kn, vn
