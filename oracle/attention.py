"""Float64 CPU oracle of the anchor-block cross-attention (test infrastructure only).

Source: *Split-KV: Efficient Context Parallelism for Training Diffusion Drafters*,
Abstract. A diffusion drafter is trained on a few draft blocks, each opened at a
sampled anchor position, whose queries cross-attend to a far longer context under
a block-sparse mask. Split-KV computes this attention without approximation while
K/V stay where they are; what moves between workers has the size of the queries.

Readings (the pages do not spell these out):

* Mask. The draft block opened by anchor ``a`` (``block`` = 16 queries) sees the
  context keys ``[0, a)`` of its own sample plus its own ``block`` keys (``Kb``,
  ``Vb`` rows of the same block), bidirectionally; no other key.
* GQA. Query head ``h`` reads kv head ``h // G`` with ``G = Hq / Hkv``.
* Scores ``s = scale * q.k`` with ``scale = 1/sqrt(d)``; ``LSE`` is the natural-log
  log-sum-exp of the scores, ``O = sum softmax(s) v``.
* Exactness with query-sized exchange means chunk-local softmax partials
  ``(O_c, LSE_c)`` combined by a log-sum-exp merge:
  ``L = log sum_c exp(LSE_c)``, ``O = sum_c exp(LSE_c - L) O_c``. An empty chunk
  contributes ``O_c = 0, LSE_c = -inf``.

Arrays are NumPy float64 views of the exact values the CUDA path receives
(bf16 inputs are upcast without change).
"""
from __future__ import annotations

from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# The core: masked softmax attention on explicit matrices.
# ---------------------------------------------------------------------------
def masked_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray,
                     mask: np.ndarray, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of rows ``q`` [R, d] over ``keys``/``values`` [N, d].

    ``mask`` [R, N] is True where a key is visible. Returns ``O`` [R, d] and the
    natural-log ``LSE`` [R]; a row with no visible key gets ``O = 0``,
    ``LSE = -inf`` (the empty-partial convention of the merge).
    """
    q = np.asarray(q, np.float64)
    keys = np.asarray(keys, np.float64)
    values = np.asarray(values, np.float64)
    s = scale * (q @ keys.T)
    s = np.where(mask, s, NEG_INF)
    R = q.shape[0]
    O = np.zeros((R, values.shape[1]))
    LSE = np.full(R, NEG_INF)
    for r in range(R):
        if not mask[r].any():
            continue
        m = s[r][mask[r]].max()
        e = np.where(mask[r], np.exp(s[r] - m), 0.0)
        total = e.sum()
        LSE[r] = m + np.log(total)
        O[r] = (e / total) @ values
    return O, LSE


def lse_merge(parts_O: List[np.ndarray], parts_LSE: List[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Exact merge of partial softmax results over disjoint key sets.

    ``L = m + log sum_c exp(LSE_c - m)`` with ``m = max_c LSE_c`` (partials with
    ``LSE = -inf`` contribute nothing); ``O = sum_c exp(LSE_c - L) O_c``. Rows
    whose partials are all empty stay ``O = 0, LSE = -inf``.
    """
    Ls = np.stack([np.asarray(x, np.float64) for x in parts_LSE])   # [C, R]
    Os = np.stack([np.asarray(x, np.float64) for x in parts_O])     # [C, R, d]
    R = Ls.shape[1]
    L = np.full(R, NEG_INF)
    O = np.zeros(Os.shape[1:])
    for r in range(R):
        live = np.isfinite(Ls[:, r])
        if not live.any():
            continue
        m = Ls[live, r].max()
        L[r] = m + np.log(np.exp(Ls[live, r] - m).sum())
        w = np.exp(Ls[live, r] - L[r])
        O[r] = (w[:, None] * Os[live, r]).sum(0)
    return O, L


# ---------------------------------------------------------------------------
# Problem bookkeeping.
# ---------------------------------------------------------------------------
class Problem:
    """The anchor-block cross-attention problem as plain arrays.

    ``anchors`` [total anchors] (ascending per sample), ``anchor_off`` [B+1],
    ``key_off`` [B+1]; ``q`` [Nq, Hq, d], ``k``/``v`` [sum S, Hkv, d],
    ``kb``/``vb`` [Nq, Hkv, d]; block ``j`` (global anchor index) owns query rows
    ``block*j .. block*j+block-1``.
    """

    def __init__(self, anchors, anchor_off, key_off, q, k, v, kb, vb, block=16, scale=None):
        self.anchors = np.asarray(anchors, np.int64)
        self.anchor_off = np.asarray(anchor_off, np.int64)
        self.key_off = np.asarray(key_off, np.int64)
        self.q = np.asarray(q, np.float64)
        self.k = np.asarray(k, np.float64)
        self.v = np.asarray(v, np.float64)
        self.kb = np.asarray(kb, np.float64)
        self.vb = np.asarray(vb, np.float64)
        self.block = int(block)
        self.Hq = self.q.shape[1]
        self.Hkv = self.k.shape[1]
        self.G = self.Hq // self.Hkv
        self.d = self.q.shape[2]
        self.scale = (1.0 / np.sqrt(self.d)) if scale is None else float(scale)
        self.B = len(self.anchor_off) - 1

    def blocks(self) -> Iterable[Tuple[int, int, int]]:
        """Yield (sample s, global block index j, anchor a)."""
        for s in range(self.B):
            for j in range(int(self.anchor_off[s]), int(self.anchor_off[s + 1])):
                yield s, j, int(self.anchors[j])

    def rows(self, j: int) -> slice:
        return slice(self.block * j, self.block * (j + 1))

    def visible(self, s: int, j: int, a: int, g: int) -> Tuple[np.ndarray, np.ndarray]:
        """Keys and values visible to block j at kv head g: context [0,a) then its own block."""
        k0 = int(self.key_off[s])
        keys = np.concatenate([self.k[k0:k0 + a, g], self.kb[self.rows(j), g]])
        vals = np.concatenate([self.v[k0:k0 + a, g], self.vb[self.rows(j), g]])
        return keys, vals


# ---------------------------------------------------------------------------
# Forward: direct single-pass definition.
# ---------------------------------------------------------------------------
def forward(p: Problem, heads: Optional[Iterable[int]] = None,
            blocks: Optional[Iterable[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """O [Nq, Hq, d] and LSE [Nq, Hq] by the plain definition.

    ``heads``/``blocks`` restrict the work to some query heads / global block
    indices (other entries stay NaN), for sampled checks at full size.
    """
    Nq = p.q.shape[0]
    O = np.full((Nq, p.Hq, p.d), np.nan)
    LSE = np.full((Nq, p.Hq), np.nan)
    hs = list(range(p.Hq)) if heads is None else list(heads)
    want = None if blocks is None else set(int(b) for b in blocks)
    for s, j, a in p.blocks():
        if want is not None and j not in want:
            continue
        r = p.rows(j)
        for h in hs:
            keys, vals = p.visible(s, j, a, h // p.G)
            mask = np.ones((p.block, keys.shape[0]), dtype=bool)
            O[r, h], LSE[r, h] = masked_attention(p.q[r, h], keys, vals, mask, p.scale)
    return O, LSE


def chunk_partials(p: Problem, chunk: int) -> Dict[Tuple[int, int, int, int], Tuple[np.ndarray, np.ndarray]]:
    """Chunk-local partials of every (sample, chunk, block, head).

    Context chunk ``c`` of a sample covers keys ``[c*chunk, min((c+1)*chunk, S))``;
    the block sees its part ``[c*chunk, min((c+1)*chunk, a))``. The block's own
    keys form one extra partial, keyed with chunk index -1. Empty partials are
    ``(0, -inf)``. Keys: ``(s, c, j, h) -> (O [block, d], LSE [block])``.
    """
    out = {}
    for s, j, a in p.blocks():
        S = int(p.key_off[s + 1] - p.key_off[s])
        n_chunks = -(-S // chunk)
        k0 = int(p.key_off[s])
        r = p.rows(j)
        for h in range(p.Hq):
            g = h // p.G
            for c in range(n_chunks):
                lo, hi = c * chunk, min((c + 1) * chunk, S)
                keys = p.k[k0 + lo:k0 + hi, g]
                vals = p.v[k0 + lo:k0 + hi, g]
                mask = np.broadcast_to(np.arange(lo, hi) < a, (p.block, hi - lo))
                out[(s, c, j, h)] = masked_attention(p.q[r, h], keys, vals, mask, p.scale)
            mask = np.ones((p.block, p.block), dtype=bool)
            out[(s, -1, j, h)] = masked_attention(p.q[r, h], p.kb[r, g], p.vb[r, g], mask, p.scale)
    return out


def merge_partials(p: Problem, parts) -> Tuple[np.ndarray, np.ndarray]:
    """Merge ``chunk_partials`` output into O [Nq, Hq, d], LSE [Nq, Hq]."""
    Nq = p.q.shape[0]
    O = np.full((Nq, p.Hq, p.d), np.nan)
    LSE = np.full((Nq, p.Hq), np.nan)
    groups: Dict[Tuple[int, int], List] = {}
    for (s, c, j, h), val in parts.items():
        groups.setdefault((j, h), []).append(val)
    for (j, h), vals in groups.items():
        r = p.rows(j)
        O[r, h], LSE[r, h] = lse_merge([x[0] for x in vals], [x[1] for x in vals])
    return O, LSE


# ---------------------------------------------------------------------------
# Backward: gradients of the same definition.
# ---------------------------------------------------------------------------
def backward(p: Problem, do: np.ndarray, O: Optional[np.ndarray] = None,
             LSE: Optional[np.ndarray] = None, blocks: Optional[Iterable[int]] = None):
    """Gradients of ``sum(O * dO)`` w.r.t. Q, K, V, Kb, Vb.

    With ``P = exp(s - LSE)`` (the softmax of each row over its visible keys),
    ``dV_j += P_j dO``, ``dP_j = dO . v_j``, ``D = sum_d dO * O``,
    ``dS_j = P_j (dP_j - D)``, ``dQ = scale sum_j dS_j k_j``,
    ``dK_j += scale dS_j q`` — the chain rule through the softmax. ``O`` and
    ``LSE`` default to this oracle's own forward. ``blocks`` restricts the sum to
    some global block indices (then dK/dV hold only their contributions), for
    sampled checks at full size. Returns
    ``(dQ [Nq,Hq,d], dK [sum S,Hkv,d], dV, dKb [Nq,Hkv,d], dVb)``.
    """
    do = np.asarray(do, np.float64)
    want = None if blocks is None else set(int(b) for b in blocks)
    if O is None or LSE is None:
        O, LSE = forward(p, blocks=want)
    dQ = np.zeros_like(p.q)
    dK = np.zeros_like(p.k)
    dV = np.zeros_like(p.v)
    dKb = np.zeros_like(p.kb)
    dVb = np.zeros_like(p.vb)
    for s, j, a in p.blocks():
        if want is not None and j not in want:
            continue
        r = p.rows(j)
        k0 = int(p.key_off[s])
        for h in range(p.Hq):
            g = h // p.G
            keys, vals = p.visible(s, j, a, g)
            qr = p.q[r, h]                      # [block, d]
            s_ = p.scale * (qr @ keys.T)        # [block, a + block]
            P = np.exp(s_ - LSE[r, h][:, None])
            dPr = do[r, h] @ vals.T
            D = (do[r, h] * O[r, h]).sum(1)
            dS = P * (dPr - D[:, None])
            dQ[r, h] += p.scale * (dS @ keys)
            dKv = p.scale * (dS.T @ qr)          # [a + block, d]
            dVv = P.T @ do[r, h]
            dK[k0:k0 + a, g] += dKv[:a]
            dV[k0:k0 + a, g] += dVv[:a]
            dKb[r, g] += dKv[a:]
            dVb[r, g] += dVv[a:]
    return dQ, dK, dV, dKb, dVb

