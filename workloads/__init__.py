"""Seeded synthetic inputs for the Split-KV hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no mask, cost, softmax or schedule). Both the CPU oracle
(through the tests) and the CUDA path consume exactly the tensors made here.

Workloads follow the shapes of *Split-KV: Efficient Context Parallelism for
Training Diffusion Drafters* (Abstract: draft blocks opened at sampled anchor
positions attend to a context far longer than the query set; the table of
target/drafter shapes: 32 query heads, 4 or 8 kv heads, head dim 128).

Draw order for one workload, from a single CPU ``torch.Generator`` seeded with
``seed``: the anchors of every sample (in sample order), then Q, K, V, Kb, Vb
and, when the workload has a backward pass, dO. Every tensor is drawn as fp32
``randn`` and then cast to the workload dtype, so both sides see the same
rounded values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import torch

__all__ = ["Workload", "WORKLOADS", "Inputs", "make_inputs", "get", "scaled"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and sampling recipe of one synthetic workload."""

    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_lens: Sequence[int]          # context length S of each sample
    anchor_counts: Sequence[int]     # anchors drawn per sample
    chunk: int                       # K/V chunk size C
    dtype: str                       # "f32" or "bf16"
    seed: int
    sampler: str = "uniform"         # "uniform" or "beta51"
    block: int = 16                  # draft block length (queries per anchor)
    key_tile: int = 128              # Tk, the key tile of the cost model
    backward: bool = False
    n_workers: Optional[int] = None  # None: one queue per SM of the device
    blocks_per_item: int = 1         # consecutive blocks sharing one query tile (128 rows on one SM, 256 on two)
    chunks_per_item: int = 1         # consecutive chunks one item covers (one partial per run of chunks)
    item_overhead: int = 0           # per-item constant of the planner's cost, in key tiles

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads of the hot path, named by what they are.
WORKLOADS = {
    w.name: w
    for w in [
        # 1 q head / 1 kv head, d=64, S=1024, 4 uniform anchors, chunk 128, fp32, 4 workers.
        Workload("tiny_f32", 1, 1, 64, [1024], [4], 128, "f32", 0, n_workers=4),
        # Drafter shape A: 32 q / 4 kv heads, d=128, S=32768, 64 anchors, chunk 1024 (items over runs of
        # 6 chunks: one partial per 6144 keys).
        Workload("drafter_s32k", 32, 4, 128, [32768], [64], 1024, "bf16", 1, chunks_per_item=6),
        # Long context: S=131072, 128 anchors, chunk 2048 (runs of 8 chunks, their cost counted in
        # 256-key tiles).
        Workload("long_s128k", 32, 4, 128, [131072], [128], 2048, "bf16", 2, chunks_per_item=8, key_tile=256),
        # Skewed anchors: 32 q / 8 kv heads, S=262144, 256 draws of floor(S*Beta(5,1)), chunk 2048.
        # G = 4: a block has 64 query rows, so two blocks share one 128-row query tile. Runs of 8 chunks
        # (one partial per 16384 keys), their cost counted in 256-key tiles (at most 64 per item).
        Workload("skewed_s256k", 32, 8, 128, [262144], [256], 2048, "bf16", 3, sampler="beta51",
                 blocks_per_item=2, chunks_per_item=8, key_tile=256),
        # Training step: 4 samples of S=65536 with 32/64/96/128 anchors, chunk 1024, fwd+bwd (runs of 8).
        Workload("train_4x64k", 32, 4, 128, [65536] * 4, [32, 64, 96, 128], 1024, "bf16", 4,
                 backward=True, chunks_per_item=8),
        # The training shape at a quarter of the context and anchors (4 x 16384 keys, 8/16/24/32
        # anchors): small enough for counter captures that replay each kernel many times.
        Workload("train_4x16k", 32, 4, 128, [16384] * 4, [8, 16, 24, 32], 1024, "bf16", 5, backward=True),
    ]
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(base: Workload, name: str, seq_lens: Sequence[int], anchor_counts: Sequence[int],
           chunk: Optional[int] = None, seed: Optional[int] = None, **kw) -> Workload:
    """A smaller workload with the same head layout, dtype and sampler as ``base``."""
    return dataclasses.replace(
        base, name=name, seq_lens=list(seq_lens), anchor_counts=list(anchor_counts),
        chunk=base.chunk if chunk is None else chunk, seed=base.seed if seed is None else seed, **kw)


@dataclasses.dataclass
class Inputs:
    """Host (CPU) tensors of one workload instance.

    Layouts (all row-major, innermost dimension last):
      anchors    int32 [total anchors]        ascending within each sample
      anchor_off int32 [B+1]                  sample s owns anchors[anchor_off[s]:anchor_off[s+1]]
      seq_len    int64 [B]
      key_off    int64 [B+1]                  sample s owns context rows key_off[s]:key_off[s+1]
      q          [Nq, Hq, d]                  Nq = block * total anchors; block b owns rows 16b..16b+15
      k, v       [sum S, Hkv, d]              packed context of all samples
      kb, vb     [Nq, Hkv, d]                 each draft block's own keys/values
      do         [Nq, Hq, d] or None          upstream gradient (backward workloads)
    """

    workload: Workload
    anchors: torch.Tensor
    anchor_off: torch.Tensor
    seq_len: torch.Tensor
    key_off: torch.Tensor
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    kb: torch.Tensor
    vb: torch.Tensor
    do: Optional[torch.Tensor]

    def anchors_of(self, s: int) -> List[int]:
        a = self.anchor_off.tolist()
        return self.anchors[a[s]:a[s + 1]].tolist()


def _draw_anchors(gen: torch.Generator, S: int, n: int, sampler: str, block: int) -> torch.Tensor:
    lo = block
    if sampler == "uniform":
        if n > S - lo:
            raise ValueError(f"cannot draw {n} distinct anchors from [{lo},{S})")
        a = torch.randperm(S - lo, generator=gen)[:n] + lo
        return torch.sort(a).values.to(torch.int32)
    if sampler == "beta51":
        # u ~ Beta(5,1) by inversion: its CDF is u^5, so u = U^(1/5) for U ~ U(0,1).
        U = torch.rand(n, generator=gen, dtype=torch.float64)
        a = torch.floor(S * U.pow(1.0 / 5.0)).to(torch.int64).clamp(lo, S - 1)
        return torch.unique(a).to(torch.int32)  # sorted, duplicates removed
    raise ValueError(f"unknown anchor sampler {sampler!r}")


def make_inputs(w: Workload) -> Inputs:
    """Draw one instance of ``w`` on the CPU, deterministically from ``w.seed``."""
    gen = torch.Generator().manual_seed(w.seed)
    anchors = [_draw_anchors(gen, int(S), int(n), w.sampler, w.block)
               for S, n in zip(w.seq_lens, w.anchor_counts)]
    counts = [int(a.numel()) for a in anchors]
    anchor_off = torch.tensor([0] + list(torch.tensor(counts).cumsum(0).tolist()), dtype=torch.int32)
    seq_len = torch.tensor([int(S) for S in w.seq_lens], dtype=torch.int64)
    key_off = torch.cat([torch.zeros(1, dtype=torch.int64), seq_len.cumsum(0)])
    n_anchor = sum(counts)
    Nq = w.block * n_anchor
    S_tot = int(key_off[-1])
    dt = w.torch_dtype

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32).to(dt)

    q = randn(Nq, w.n_q_heads, w.head_dim)
    k = randn(S_tot, w.n_kv_heads, w.head_dim)
    v = randn(S_tot, w.n_kv_heads, w.head_dim)
    kb = randn(Nq, w.n_kv_heads, w.head_dim)
    vb = randn(Nq, w.n_kv_heads, w.head_dim)
    do = randn(Nq, w.n_q_heads, w.head_dim) if w.backward else None
    return Inputs(w, torch.cat(anchors) if anchors else torch.zeros(0, dtype=torch.int32),
                  anchor_off, seq_len, key_off, q, k, v, kb, vb, do)
