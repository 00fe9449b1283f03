"""Split-KV context parallelism across GPUs (one rank per GPU, ``torch.distributed`` for the exchange).

*Split-KV: Efficient Context Parallelism for Training Diffusion Drafters*, Abstract and its table of
context-parallel methods: every rank keeps a global view of the (short) draft query set, the context
K/V chunks are placed on ranks by a cost-aware longest-processing-time-first plan on their realized
attention cost, K/V never leave the rank that owns them, and the only per-layer attention exchange is
of query-sized tensors, so it does not grow with the context length.

One forward on rank r of n (every step runs in ``libsplitkv.so``; this module only orders the calls and
the collective):

1. ``plan``: the chunk costs (``splitkv_cost``, the same on every rank since every rank has all anchors)
   are copied to the host and placed by ``splitkv_cp_plan`` (host LPT; identical on every rank, so no
   message is needed); this rank's items (``splitkv_cost_rank``) are then planned onto this GPU's SMs
   (``splitkv_plan_lpt``).
2. ``local_forward``: this rank's chunk partials (``splitkv_attn_fwd``) merged into one query-sized
   ``(O_r, LSE_r)`` (``splitkv_lse_merge_rank``).
3. ``gather``: an all-gather of ``(O_r, LSE_r)`` over the group: ``n * Nq * Hq * (d + 1)`` values.
4. ``combine``: the exact log-sum-exp merge over ranks (``splitkv_lse_merge_ranks``), equal to the
   single-GPU result.

One backward on rank r, from the merged O and LSE (which every rank holds after ``combine``):

5. ``local_backward``: this rank's share (``splitkv_attn_bwd_rank``): dK/dV of its chunks' keys, final as
   they are (K/V never leave the rank), and partial dQ, dKb, dVb (its keys, its blocks' own keys);
6. ``reduce_grads``: one all-reduce (sum) of dQ, dKb and dVb over the group: ``Nq * (Hq + 2 Hkv) * d``
   values, again independent of the context length.

K/V layout: each rank passes full-size ``k``/``v`` buffers ([sum S, Hkv, d]) of which only the rows of its
own chunks are read (the others may hold anything); a compact per-rank layout would need a chunk-to-row
map in the kernels and is not built. Items cover one chunk each (``chunks_per_item`` = 1).
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


def reduce_rank_grads(dq, dkb, dvb, group=None):
    """Sums this rank's partial dQ, dKb and dVb over ``group`` in place (one all-reduce of the three,
    packed into one buffer): after it every rank holds the single-GPU gradients of the query side."""
    import torch.distributed as dist
    flat = torch.cat([dq.reshape(-1), dkb.reshape(-1), dvb.reshape(-1)])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    a, b = dq.numel(), dkb.numel()
    dq.copy_(flat[:a].view_as(dq))
    dkb.copy_(flat[a:a + b].view_as(dkb))
    dvb.copy_(flat[a + b:].view_as(dvb))
    return dq, dkb, dvb


def cp_plan_chunks(chunk_cost, n_ranks: int):
    """Chunk -> rank by the host LPT (``splitkv_cp_plan``): ``(chunk_rank, rank_load)`` CPU tensors."""
    return B.splitkv_cp_plan(chunk_cost, n_ranks)


def gather_rank_results(o_r: torch.Tensor, lse_r: torch.Tensor, group=None):
    """All-gather of this rank's query-sized result over ``group``: ``([n, *o_r.shape], [n, *lse_r.shape])``
    in rank order (the only exchange of the forward)."""
    import torch.distributed as dist
    n = dist.get_world_size(group)
    # Gathered along dim 0 (the ranks' tensors one after another), then viewed per rank.
    o_all = torch.empty((n * o_r.shape[0],) + tuple(o_r.shape[1:]), dtype=o_r.dtype, device=o_r.device)
    lse_all = torch.empty((n * lse_r.shape[0],) + tuple(lse_r.shape[1:]), dtype=lse_r.dtype, device=lse_r.device)
    dist.all_gather_into_tensor(o_all, o_r.contiguous(), group=group)
    dist.all_gather_into_tensor(lse_all, lse_r.contiguous(), group=group)
    return o_all.view((n,) + tuple(o_r.shape)), lse_all.view((n,) + tuple(lse_r.shape))


class ContextParallelSplitKV:
    """Buffers and calls of one rank for one problem shape (see the module docstring).

    ``rank``/``n_ranks`` default to the process group's; they can be given explicitly to run the ranks'
    steps one after another on one GPU (the all-gather is then the caller's).
    """

    def __init__(self, seq_lens, anchor_counts, n_q_heads, n_kv_heads, head_dim, block=16, chunk=1024,
                 key_tile=128, scale=None, dtype=torch.bfloat16, n_workers=None, device="cuda", blocks_per_item=1,
                 group=None, rank: Optional[int] = None, n_ranks: Optional[int] = None):
        if rank is None or n_ranks is None:
            import torch.distributed as dist
            rank, n_ranks = dist.get_rank(group), dist.get_world_size(group)
        self.group, self.rank, self.n_ranks = group, int(rank), int(n_ranks)
        self.skv = B.SplitKV(seq_lens, anchor_counts, n_q_heads, n_kv_heads, head_dim, block, chunk, key_tile, scale,
                             dtype, n_workers=n_workers, device=device, blocks_per_item=blocks_per_item)
        self.chunk_rank = None   # device int32[n_chunks]
        self.rank_load = None    # host int64[n_ranks]

    def plan(self, anchors, stream=None):
        skv = self.skv
        skv.cost(anchors, stream)  # chunk costs of every chunk
        chunk_cost = skv.chunk_cost[: int(skv.sizes.n_chunks)].cpu()  # synchronizes with the stream
        chunk_rank, self.rank_load = cp_plan_chunks(chunk_cost, self.n_ranks)
        self.chunk_rank = chunk_rank.to(skv.device)
        B.splitkv_cost_rank(skv.problem, anchors, self.chunk_rank, self.rank, self.n_ranks, skv.item_id,
                            skv.item_cost, skv.chunk_cost, skv.n_items, skv.status, skv.workspace, stream)
        skv.plan_lpt(stream)

    def local_forward(self, q, k, v, kb, vb, anchors, stream=None):
        """This rank's (O_r, LSE_r): the partials of its chunks (and of its share of the blocks' own keys)."""
        skv = self.skv
        skv.attn_fwd(q, k, v, kb, vb, anchors, stream=stream)
        Nq, Hq, d = int(skv.sizes.n_queries), skv.n_q_heads, skv.head_dim
        o_r = torch.empty(Nq, Hq, d, dtype=skv.dtype, device=skv.device)
        lse_r = torch.empty(Nq, Hq, dtype=torch.float32, device=skv.device)
        B.splitkv_lse_merge_rank(skv.problem, skv.o_part, skv.lse_part, anchors, self.chunk_rank, self.rank,
                                 self.n_ranks, o_r, lse_r, skv.status, stream)
        return o_r, lse_r

    def combine(self, o_ranks, lse_ranks, stream=None):
        """Exact merge of the ranks' results ([n_ranks, Nq, Hq, d], [n_ranks, Nq, Hq]) into (O, LSE)."""
        skv = self.skv
        o = torch.empty(o_ranks.shape[1:], dtype=skv.dtype, device=skv.device)
        lse = torch.empty(lse_ranks.shape[1:], dtype=torch.float32, device=skv.device)
        B.splitkv_lse_merge_ranks(skv.problem, int(o_ranks.shape[0]), o_ranks, lse_ranks, o, lse, skv.status, stream)
        return o, lse

    def forward(self, q, k, v, kb, vb, anchors, stream=None):
        self.plan(anchors, stream)
        o_r, lse_r = self.local_forward(q, k, v, kb, vb, anchors, stream)
        o_all, lse_all = gather_rank_results(o_r, lse_r, self.group)
        return self.combine(o_all, lse_all, stream)

    def local_backward(self, q, k, v, kb, vb, o, lse, dout, anchors, stream=None):
        """This rank's share of the gradients (float32): dk, dv on its chunks' key rows (zero elsewhere),
        partial dq, dkb, dvb. Needs the chunk placement of the last :meth:`plan`."""
        skv = self.skv
        f = dict(dtype=torch.float32, device=skv.device)
        dq, dk, dv = torch.empty(q.shape, **f), torch.empty(k.shape, **f), torch.empty(v.shape, **f)
        dkb, dvb = torch.empty(kb.shape, **f), torch.empty(vb.shape, **f)
        B.splitkv_attn_bwd_rank(skv.problem, q, k, v, kb, vb, o, lse, dout, anchors, self.chunk_rank, self.rank,
                                self.n_ranks, dq, dk, dv, dkb, dvb, skv.status, skv.workspace, stream)
        return dq, dk, dv, dkb, dvb

    def backward(self, q, k, v, kb, vb, o, lse, dout, anchors, stream=None):
        dq, dk, dv, dkb, dvb = self.local_backward(q, k, v, kb, vb, o, lse, dout, anchors, stream)
        reduce_rank_grads(dq, dkb, dvb, self.group)
        return dq, dk, dv, dkb, dvb
