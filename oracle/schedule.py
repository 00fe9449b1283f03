"""Integer oracle of the realized chunk cost and the cost-aware LPT plan (test infrastructure only).

Source: *Split-KV: Efficient Context Parallelism for Training Diffusion Drafters*,
Abstract. Since every worker knows all draft queries, the work of each context
chunk can be counted before attention runs, and a longest-processing-time-first
(LPT) greedy places chunks by that count; with anchor sampling the count changes
from sample to sample and is not linear in the chunk's position.
The page's table of context-parallel methods names cost-aware LPT as Split-KV's load balancing.

Readings (the pages give neither the cost unit nor the LPT details):

* Work item = (sample s, chunk c, kv head g, block b). Its query tile is the
  ``block * G`` rows of block b at the G query heads of kv head g; its key tiles
  are the ``key_tile`` (Tk, 128 unless a workload counts coarser tiles) slices of chunk c. Item cost = number of key
  tiles holding at least one key the block sees; items of cost 0 are dropped.
* Item index (chunk-major): ``base_s + (c * Hkv + g) * n_blocks_s + b`` where
  ``base_s`` counts the items of earlier samples and ``n_chunks_s = ceil(S/C)``.
* Chunk cost = sum of the costs of that chunk's items.
* Query tiles of several blocks (``pack`` = P >= 1, default 1). With P > 1 an item
  is (s, c, g, t): the query tile holds blocks ``tP .. min(tP+P, n_blocks_s) - 1``
  of sample s (their rows stacked, each row masked by its own block's anchor), and
  its cost counts the key tiles that any of those rows sees. P = 1 is the item of
  the lines above. Index: ``base_s + (c * Hkv + g) * ceil(n_blocks_s / P) + t``.
* Runs of chunks (``runs`` = L >= 1, default 1). With L > 1 an item covers the L
  consecutive chunks ``rL .. rL+L-1`` of its sample (run r: keys ``[rLC, min((r+1)LC, S))``),
  so one worker carries the softmax of a query tile across them and leaves one partial
  per run. Its cost counts the key tiles of the run that any of its rows sees; the chunk
  cost stays per chunk of C keys (the sum over items of their tiles inside that chunk),
  so it does not depend on L. Index: ``base_s + (r * Hkv + g) * n_tiles_s + t`` with
  ``ceil(ceil(S/C) / L)`` runs. L = 1 is the item of the lines above.
* Per-item constant (``overhead`` = kappa >= 0, default 0). The realized cost of a visible
  item may add a fixed kappa (in key-tile units) for the work every item carries whatever
  its length (loading its query tile, writing its partial): cost = tiles + kappa. Chunk
  costs count key tiles only. kappa = 0 is the item cost of the lines above.
* LPT: order items by (cost descending, item index ascending); give each in turn
  to the worker with the least (load, worker index); loads start at 0; a
  worker's queue lists its items in assignment order.
* Imbalance = max(load) / mean(load) - 1.
"""
from __future__ import annotations

import heapq
import itertools
from typing import Dict, List, Sequence, Tuple

import numpy as np


def item_layout(anchor_counts: Sequence[int], seq_lens: Sequence[int], chunk: int, n_kv_heads: int,
                pack: int = 1, runs: int = 1):
    """Per-sample (base item index, n_item_chunks, n_query_tiles) and the total item count; an item
    chunk is a run of ``runs`` chunks (the last one of a sample may be shorter)."""
    out = []
    base = 0
    for nb, S in zip(anchor_counts, seq_lens):
        nc = -(-(-(-int(S) // chunk)) // runs)
        nt = -(-int(nb) // pack)
        out.append((base, nc, nt))
        base += nc * n_kv_heads * nt
    return out, base


def costs_bruteforce(anchors_per_sample: Sequence[Sequence[int]], seq_lens: Sequence[int], chunk: int,
                     key_tile: int, n_kv_heads: int, group: int, block: int = 16, pack: int = 1, runs: int = 1,
                     overhead: int = 0):
    """Item costs by enumerating the boolean mask of every (query tile, key tile).

    Returns ``(item_ids, item_costs, chunk_costs)``: visible items in ascending
    index order, their costs, and per-(sample, chunk) costs (flattened, sample-major;
    a chunk is ``chunk`` keys whatever ``runs`` is). For small inputs only.
    """
    layout, _ = item_layout([len(a) for a in anchors_per_sample], seq_lens, chunk, n_kv_heads, pack, runs)
    span = chunk * runs  # keys of an item chunk (a run of chunks)
    ids, costs, chunk_costs = [], [], []
    for s, anchors in enumerate(anchors_per_sample):
        base, nr, nt = layout[s]
        S = int(seq_lens[s])
        per_chunk = np.zeros(-(-S // chunk), np.int64)
        for r in range(nr):
            lo, hi = r * span, min((r + 1) * span, S)
            keys = np.arange(lo, hi)
            for g in range(n_kv_heads):
                for t in range(nt):
                    # rows of every block of the tile; a row sees context key k iff k < its block's anchor
                    members = anchors[t * pack:(t + 1) * pack]
                    mask = np.concatenate([np.broadcast_to(keys < a, (block * group, hi - lo)) for a in members])
                    n_tiles = -(-(hi - lo) // key_tile)
                    cost = 0
                    for kt in range(n_tiles):
                        if mask[:, kt * key_tile:(kt + 1) * key_tile].any():
                            cost += 1
                            per_chunk[(lo + kt * key_tile) // chunk] += 1  # the chunk holding this key tile
                    if cost:
                        ids.append(base + (r * n_kv_heads + g) * nt + t)
                        costs.append(cost + overhead)
        chunk_costs.extend(per_chunk.tolist())
    return np.array(ids, np.int64), np.array(costs, np.int64), np.array(chunk_costs, np.int64)


def costs_closed_form(anchors_per_sample, seq_lens, chunk, key_tile, n_kv_heads, pack: int = 1, runs: int = 1,
                      overhead: int = 0):
    """Same result in closed form: ``cost = ceil(clamp(a - r*LC, 0, min(LC, S - r*LC)) / Tk)`` over the
    item's run of L = ``runs`` chunks, with ``a`` the largest anchor of the item's blocks (the last
    one: anchors ascend); chunk c's cost sums ``ceil(clamp(a - c*C, 0, min(C, S - c*C)) / Tk)`` over
    the tiles and kv heads (key tiles never straddle a chunk: C is a multiple of Tk)."""
    layout, _ = item_layout([len(a) for a in anchors_per_sample], seq_lens, chunk, n_kv_heads, pack, runs)
    span = chunk * runs
    ids, costs, chunk_costs = [], [], []
    for s, anchors in enumerate(anchors_per_sample):
        base, nr, nt = layout[s]
        S = int(seq_lens[s])
        a = np.asarray(anchors, np.int64)
        a_last = np.array([a[min((t + 1) * pack, len(a)) - 1] for t in range(nt)], np.int64)
        for r in range(nr):
            width = min(span, S - r * span)
            cost = -(-np.clip(a_last - r * span, 0, width) // key_tile)
            for g in range(n_kv_heads):
                for t in range(nt):
                    if cost[t]:
                        ids.append(base + (r * n_kv_heads + g) * nt + t)
                        costs.append(int(cost[t]) + overhead)
        for c in range(-(-S // chunk)):
            width = min(chunk, S - c * chunk)
            chunk_costs.append(int(n_kv_heads * np.sum(-(-np.clip(a_last - c * chunk, 0, width) // key_tile))))
    return np.array(ids, np.int64), np.array(costs, np.int64), np.array(chunk_costs, np.int64)


def lpt(costs: Sequence[int], n_workers: int):
    """Longest-processing-time-first greedy, with a binary heap of (load, worker).

    Returns ``(item_worker, queue_off, queue_items, load)``: the worker of each
    item (items indexed by position in ``costs``), the queues in CSR form (each
    in assignment order), and the final loads.
    """
    costs = [int(c) for c in costs]
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    heap = [(0, w) for w in range(n_workers)]
    heapq.heapify(heap)
    item_worker = [-1] * len(costs)
    queues: List[List[int]] = [[] for _ in range(n_workers)]
    for i in order:
        load, w = heapq.heappop(heap)
        item_worker[i] = w
        queues[w].append(i)
        heapq.heappush(heap, (load + costs[i], w))
    load = [0] * n_workers
    for i, w in enumerate(item_worker):
        load[w] += costs[i]
    queue_off = [0]
    for q in queues:
        queue_off.append(queue_off[-1] + len(q))
    queue_items = [i for q in queues for i in q]
    return (np.array(item_worker, np.int64), np.array(queue_off, np.int64),
            np.array(queue_items, np.int64), np.array(load, np.int64))


def naive_split(costs: Sequence[int], n_workers: int):
    """Cost-blind equal-count split: item list (index order) cut into contiguous pieces.

    Worker ``w`` gets items ``[floor(w*n/m), floor((w+1)*n/m))``. Returns the same
    tuple as :func:`lpt`.
    """
    n = len(costs)
    bounds = [(w * n) // n_workers for w in range(n_workers + 1)]
    item_worker = np.zeros(n, np.int64)
    load = np.zeros(n_workers, np.int64)
    for w in range(n_workers):
        item_worker[bounds[w]:bounds[w + 1]] = w
        load[w] = int(np.sum(np.asarray(costs[bounds[w]:bounds[w + 1]], np.int64)))
    return item_worker, np.array(bounds, np.int64), np.arange(n, dtype=np.int64), load


def makespan(load) -> int:
    return int(np.max(load)) if len(load) else 0


def imbalance(load) -> float:
    """max(load) / mean(load) - 1 (0 for an empty plan)."""
    load = np.asarray(load, np.float64)
    if load.size == 0 or load.sum() == 0:
        return 0.0
    return float(load.max() / load.mean() - 1.0)


def optimal_makespan(costs: Sequence[int], n_workers: int) -> int:
    """Exhaustive minimum makespan over all n_workers^n assignments (tiny inputs)."""
    costs = [int(c) for c in costs]
    best = None
    for assign in itertools.product(range(n_workers), repeat=len(costs)):
        loads = [0] * n_workers
        for c, w in zip(costs, assign):
            loads[w] += c
        mk = max(loads) if loads else 0
        if best is None or mk < best:
            best = mk
    return 0 if best is None else best
