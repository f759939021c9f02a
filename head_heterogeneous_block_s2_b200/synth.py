"""Seeded synthetic inputs for HHST sparse attention (shared by tests, smoke and bench).

This module holds no attention arithmetic: it only draws random tensors, rounds
them to bf16 and lays them out (dense [batch, heads, seq, D] tensors for
prefill; a paged cache with a permuted block table for decode). Both the CUDA
path and the CPU oracle receive exactly the tensors made here.

Workloads (the pages train 1.3B and 7B HHST models and claim retrieval at a
128K context and serving through a paged KV cache; they print no shapes, so the
sizes below are the build's chosen stand-ins for those settings):

====================  =====================================================
tiny                  batch 1, 4 heads, D 64, seq 512, B 64, S 4, L 1
prefill_1p3b          batch 4, 16 heads, D 128, seq 8192, B 64, S 8, L 2;
                      K of head h multiplied by a per-head U(0.5, 2) scalar
prefill_7b_hybrid     batch 1, 32 heads, D 128, seq 32768, B 128, S 16, L 4;
                      heads 0-3 dense causal
prefill_long_131k     batch 1, 32 heads, D 128, seq 131072, B 128, S 16, L 4;
                      one planted key row per head (a copy of 2x the last query)
decode_paged          batch 64, 32 heads, D 128, context U[4096, 32768],
                      16-token pages, permuted block table, B 128, S 16, L 4
====================  =====================================================

Draw order for one workload (a torch.Generator seeded with ``seed``):
prefill: Q, K, V (each N(0,1) fp32), then the per-head K scales when present;
K is scaled in fp32 before rounding. Decode: context lengths, the page
permutation, then q, the K cache and the V cache. Everything is rounded to bf16
with round-to-nearest-even (torch's fp32 -> bf16 conversion).
"""
from __future__ import annotations

import dataclasses
import itertools
import math
from typing import Dict, Optional, Sequence, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    batch: int
    heads: int
    head_dim: int
    seq: int
    block: int  # B: tokens per block (query and key)
    stride: int  # S: vertical stride
    local: int  # L: local blocks
    dense_heads: Tuple[int, ...] = ()
    seed: int = 0
    k_scale_range: Optional[Tuple[float, float]] = None
    planted: bool = False

    @property
    def num_blocks(self) -> int:
        return -(-self.seq // self.block)  # a ragged last block counts

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def with_(self, **kw) -> "PrefillWorkload":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    heads: int
    head_dim: int
    ctx_min: int
    ctx_max: int  # inclusive
    page_size: int
    block: int
    stride: int
    local: int
    dense_heads: Tuple[int, ...] = ()
    seed: int = 4

    @property
    def max_pages(self) -> int:
        return -(-self.ctx_max // self.page_size)

    @property
    def num_blocks(self) -> int:
        return -(-self.ctx_max // self.block)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def with_(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


TINY = PrefillWorkload("tiny", 1, 4, 64, 512, 64, 4, 1, seed=0)
PREFILL_1P3B = PrefillWorkload("prefill_1p3b", 4, 16, 128, 8192, 64, 8, 2, seed=1,
                               k_scale_range=(0.5, 2.0))
PREFILL_7B_HYBRID = PrefillWorkload("prefill_7b_hybrid", 1, 32, 128, 32768, 128, 16, 4,
                                    dense_heads=(0, 1, 2, 3), seed=2)
PREFILL_LONG_131K = PrefillWorkload("prefill_long_131k", 1, 32, 128, 131072, 128, 16, 4,
                                    seed=3, planted=True)
DECODE_PAGED = DecodeWorkload("decode_paged", 64, 32, 128, 4096, 32768, 16, 128, 16, 4, seed=4)

# Chunked prefill over the paged cache (serving): 16 sequences with contexts
# U[4096, 32768], each ending in a chunk of the last 2048 tokens; same pattern
# and page layout as decode_paged.
CHUNK_PAGED = DecodeWorkload("chunk_paged", 16, 32, 128, 4096, 32768, 16, 128, 16, 4, seed=5)
CHUNK_LEN = {"chunk_paged": 2048}

PREFILL_WORKLOADS = {w.name: w for w in (TINY, PREFILL_1P3B, PREFILL_7B_HYBRID, PREFILL_LONG_131K)}
DECODE_WORKLOADS = {DECODE_PAGED.name: DECODE_PAGED}
CHUNK_WORKLOADS = {CHUNK_PAGED.name: CHUNK_PAGED}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def _normal_bf16(shape, g, device, chunk_elems: int = 1 << 28) -> torch.Tensor:
    """N(0,1) drawn in fp32 and rounded to bf16, in chunks to bound fp32 scratch."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk_elems):
        e = min(flat.numel(), s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=g, device=device, dtype=torch.float32)
    return out


def prefill_inputs(w: PrefillWorkload, device="cpu",
                   plant_positions: Optional[Dict[int, int]] = None):
    """Q, K, V bf16 [batch, heads, seq, head_dim] for workload ``w``.

    plant_positions: optional {head: token} map. For each entry, K[:, head, token]
    is set to 2 x Q[:, head, seq-1] (exact in bf16: a power-of-two multiple).
    The caller chooses the tokens (the generator knows nothing of the pattern).
    """
    shape = (w.batch, w.heads, w.seq, w.head_dim)
    g = _gen(w.seed, device)
    q = _normal_bf16(shape, g, device)
    if w.k_scale_range is None:
        k = _normal_bf16(shape, g, device)
        v = _normal_bf16(shape, g, device)
    else:
        kf = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        v = _normal_bf16(shape, g, device)
        lo, hi = w.k_scale_range
        sc = lo + (hi - lo) * torch.rand(w.heads, generator=g, device=device, dtype=torch.float32)
        k = (kf * sc.view(1, -1, 1, 1)).to(torch.bfloat16)
        del kf
    if plant_positions:
        for h, t in plant_positions.items():
            k[:, h, t, :] = q[:, h, w.seq - 1, :] * 2
    return q, k, v


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor  # bf16 [batch, heads, D]
    k_cache: torch.Tensor  # bf16 [num_pages, heads, page_size, D]
    v_cache: torch.Tensor
    block_table: torch.Tensor  # int32 [batch, max_pages], -1 padded
    ctx_lens: torch.Tensor  # int32 [batch]

    @property
    def num_pages(self) -> int:
        return self.k_cache.shape[0]


def decode_inputs(w: DecodeWorkload, device="cpu", ctx_lens: Optional[Sequence[int]] = None,
                  page_chunk: int = 4096) -> DecodeInputs:
    """Paged decode inputs for ``w``.

    Context lengths are U[ctx_min, ctx_max] integers (unless given). Physical
    page ids are a seeded permutation of 0..num_pages-1, handed to the
    sequences' logical pages in order; unused block-table slots hold -1.
    """
    g = _gen(w.seed, device)
    if ctx_lens is None:
        cl = torch.randint(w.ctx_min, w.ctx_max + 1, (w.batch,), generator=g, device=device,
                           dtype=torch.int64)
    else:
        cl = torch.tensor(list(ctx_lens), dtype=torch.int64, device=device)
    cl_host = cl.cpu()
    pages_per_seq = [(-(-int(n) // w.page_size)) for n in cl_host.tolist()]
    num_pages = sum(pages_per_seq)
    perm = torch.randperm(num_pages, generator=g, device=device).to(torch.int32).cpu()
    max_pages = max(w.max_pages, max(pages_per_seq))
    bt = torch.full((w.batch, max_pages), -1, dtype=torch.int32)
    off = 0
    for s, n in enumerate(pages_per_seq):
        bt[s, :n] = perm[off:off + n]
        off += n
    q = _normal_bf16((w.batch, w.heads, w.head_dim), g, device)
    shape = (num_pages, w.heads, w.page_size, w.head_dim)
    k_cache = torch.empty(shape, dtype=torch.bfloat16, device=device)
    v_cache = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for cache in (k_cache, v_cache):
        for p0 in range(0, num_pages, page_chunk):
            p1 = min(num_pages, p0 + page_chunk)
            cache[p0:p1] = torch.randn((p1 - p0,) + shape[1:], generator=g, device=device,
                                       dtype=torch.float32)
    return DecodeInputs(q, k_cache, v_cache, bt.to(device), cl.to(torch.int32).to(device))


@dataclasses.dataclass
class ChunkInputs:
    q: torch.Tensor            # [total_q, heads, head_dim] packed chunk rows
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_table: torch.Tensor
    ctx_lens: torch.Tensor     # contexts including the chunks
    q_start: torch.Tensor      # [batch + 1]
    max_q_len: int


def chunk_inputs(w: DecodeWorkload, chunk: int, device="cpu") -> ChunkInputs:
    """Chunked-prefill inputs: the paged contexts of ``w`` (as decode_inputs)
    and, per sequence, a chunk of its last min(chunk, context) tokens as
    packed N(0,1) query rows."""
    d = decode_inputs(w, device=device)
    cl = d.ctx_lens.cpu().tolist()
    qlen = [min(chunk, n) for n in cl]
    q_start = torch.tensor([0] + list(itertools.accumulate(qlen)), dtype=torch.int32)
    g = _gen(w.seed + 1000, device)
    q = _normal_bf16((int(q_start[-1]), w.heads, w.head_dim), g, device)
    return ChunkInputs(q, d.k_cache, d.v_cache, d.block_table, d.ctx_lens, q_start.to(device), max(qlen))
