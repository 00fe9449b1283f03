"""Pins of the float64 attention oracle against facts other than itself.

* torch's scaled_dot_product_attention (float64, CPU) on an explicit boolean mask,
  and torch.logsumexp of the explicitly masked score matrix;
* closed forms: Q = 0 gives a uniform softmax; constant V returns the constant;
  a single visible key returns its value row and its own score;
* the exact merge: any split of the keys into partials merges back to the
  single pass, in any order;
* torch.autograd (float64) and central finite differences for the gradients,
  and the softmax invariants sum_j dK_j = 0, sum_j dV_j = sum_rows dO.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import attention as A
from tests._util import oracle_problem, to_np

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def tiny(name="t", seq_lens=(96, 160), counts=(3, 4), hq=4, hkv=2, d=16, chunk=32, seed=7,
         sampler="uniform", block=16):
    base = workloads.Workload(name, hq, hkv, d, list(seq_lens), list(counts), chunk, "f32", seed,
                              sampler=sampler, block=block, key_tile=16, backward=True)
    return workloads.make_inputs(base)


def dense_mask_problem(inp, s):
    """Per sample: all context keys then every block's own keys, with the explicit mask."""
    w = inp.workload
    a = inp.anchors_of(s)
    ao = inp.anchor_off.tolist()
    ko = inp.key_off.tolist()
    rows = slice(w.block * ao[s], w.block * ao[s + 1])
    S = ko[s + 1] - ko[s]
    nq = w.block * len(a)
    keys = torch.cat([inp.k[ko[s]:ko[s + 1]], inp.kb[rows]]).double()     # [S+nq, Hkv, d]
    vals = torch.cat([inp.v[ko[s]:ko[s + 1]], inp.vb[rows]]).double()
    mask = torch.zeros(nq, S + nq, dtype=torch.bool)
    for b, anc in enumerate(a):
        r = slice(w.block * b, w.block * (b + 1))
        mask[r, :anc] = True
        mask[r, S + w.block * b:S + w.block * (b + 1)] = True
    return rows, keys, vals, mask


def torch_reference(inp, q=None, k=None, v=None, kb=None, vb=None):
    """Forward through torch ops on the explicit masks (one sample at a time)."""
    w = inp.workload
    G = w.group
    q = inp.q.double() if q is None else q
    outs, lses = [], []
    for s in range(len(w.seq_lens)):
        rows, keys, vals, mask = dense_mask_problem(inp, s)
        if k is not None:
            ao, ko = inp.anchor_off.tolist(), inp.key_off.tolist()
            keys = torch.cat([k[ko[s]:ko[s + 1]], kb[rows]])
            vals = torch.cat([v[ko[s]:ko[s + 1]], vb[rows]])
        qh = q[rows].permute(1, 0, 2)                                       # [Hq, nq, d]
        kh = keys.permute(1, 0, 2).repeat_interleave(G, 0)                  # [Hq, N, d]
        vh = vals.permute(1, 0, 2).repeat_interleave(G, 0)
        o = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask, scale=w.scale)
        sc = (qh @ kh.transpose(1, 2)) * w.scale
        lse = torch.logsumexp(sc.masked_fill(~mask, float("-inf")), dim=-1)
        outs.append(o.permute(1, 0, 2))
        lses.append(lse.permute(1, 0))
    return torch.cat(outs), torch.cat(lses)


@pytest.mark.parametrize("kw", [dict(), dict(hq=2, hkv=2), dict(hq=8, hkv=1, d=8), dict(block=4, counts=(5, 2))])
def test_forward_matches_sdpa_on_explicit_mask(kw):
    inp = tiny(**kw)
    O, L = A.forward(oracle_problem(inp))
    O_ref, L_ref = torch_reference(inp)
    np.testing.assert_allclose(O, O_ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, L_ref.numpy(), rtol=0, atol=1e-12)


def test_zero_query_is_uniform_softmax():
    inp = tiny()
    inp.q.zero_()
    p = oracle_problem(inp)
    O, L = A.forward(p)
    w = inp.workload
    for s, j, a in p.blocks():
        r = p.rows(j)
        assert np.allclose(L[r], math.log(a + w.block), atol=1e-13)
        for h in range(w.n_q_heads):
            g = h // w.group
            ko = int(inp.key_off[s])
            rows_v = [to_np(inp.v[ko + t, g]) for t in range(a)] + \
                     [to_np(inp.vb[w.block * j + t, g]) for t in range(w.block)]
            mean = sum(rows_v) / len(rows_v)
            assert np.allclose(O[r, h], mean[None, :], atol=1e-13)


def test_constant_values_return_the_constant():
    inp = tiny()
    inp.v.fill_(0.75)
    inp.vb.fill_(0.75)
    O, _ = A.forward(oracle_problem(inp))
    assert np.allclose(O, 0.75, atol=1e-14)


def test_single_visible_key_returns_its_row_and_score(rng):
    q = rng.standard_normal((3, 8))
    keys = rng.standard_normal((5, 8))
    vals = rng.standard_normal((5, 8))
    mask = np.zeros((3, 5), dtype=bool)
    mask[0, 2] = True
    mask[1, 4] = True
    O, L = A.masked_attention(q, keys, vals, mask, 0.5)
    assert np.allclose(O[0], vals[2]) and np.isclose(L[0], 0.5 * q[0] @ keys[2])
    assert np.allclose(O[1], vals[4]) and np.isclose(L[1], 0.5 * q[1] @ keys[4])
    assert np.all(O[2] == 0) and L[2] == -np.inf  # no visible key: empty partial


@pytest.mark.parametrize("chunk", [16, 32, 48, 1000])
def test_chunk_partials_merge_to_single_pass(chunk):
    inp = tiny(seq_lens=(100, 64), counts=(4, 2))  # 100 % 16 != 0: ragged tail chunk
    p = oracle_problem(inp)
    O, L = A.forward(p)
    Om, Lm = A.merge_partials(p, A.chunk_partials(p, chunk))
    np.testing.assert_allclose(Om, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(Lm, L, rtol=0, atol=1e-13)


def test_merge_is_order_free_and_skips_empty(rng):
    q = rng.standard_normal((4, 8))
    keys = rng.standard_normal((30, 8))
    vals = rng.standard_normal((30, 8))
    full = np.ones((4, 30), dtype=bool)
    O, L = A.masked_attention(q, keys, vals, full, 0.3)
    cuts = [0, 7, 8, 19, 30]
    parts = [A.masked_attention(q, keys[a:b], vals[a:b], full[:, a:b], 0.3) for a, b in zip(cuts, cuts[1:])]
    parts.append((np.zeros((4, 8)), np.full(4, -np.inf)))  # an empty partial changes nothing
    for perm in ([0, 1, 2, 3, 4], [4, 2, 0, 3, 1]):
        Om, Lm = A.lse_merge([parts[i][0] for i in perm], [parts[i][1] for i in perm])
        np.testing.assert_allclose(Om, O, atol=1e-14)
        np.testing.assert_allclose(Lm, L, atol=1e-14)
    Oe, Le = A.lse_merge([np.zeros((4, 8))], [np.full(4, -np.inf)])
    assert np.all(Oe == 0) and np.all(Le == -np.inf)


@pytest.mark.parametrize("kw", [dict(), dict(hq=8, hkv=1, d=8, counts=(2, 3))])
def test_backward_matches_autograd(kw):
    inp = tiny(**kw)
    p = oracle_problem(inp)
    do = to_np(inp.do)
    dQ, dK, dV, dKb, dVb = A.backward(p, do)
    ts = [t.double().clone().requires_grad_(True) for t in (inp.q, inp.k, inp.v, inp.kb, inp.vb)]
    O_ref, _ = torch_reference(inp, *ts)
    (O_ref * inp.do.double()).sum().backward()
    for mine, t in zip((dQ, dK, dV, dKb, dVb), ts):
        np.testing.assert_allclose(mine, t.grad.numpy(), rtol=0, atol=1e-12)


def test_backward_finite_differences(rng):
    inp = tiny(seq_lens=(40,), counts=(2,), hq=2, hkv=1, d=4, block=3)
    p = oracle_problem(inp)
    do = to_np(inp.do)
    grads = A.backward(p, do)
    names = ("q", "k", "v", "kb", "vb")
    eps = 1e-6
    for name, grad in zip(names, grads):
        arr = getattr(p, name)
        for _ in range(4):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            old = arr[idx]
            arr[idx] = old + eps
            fp = (A.forward(p)[0] * do).sum()
            arr[idx] = old - eps
            fm = (A.forward(p)[0] * do).sum()
            arr[idx] = old
            assert abs((fp - fm) / (2 * eps) - grad[idx]) < 1e-6, (name, idx)


def test_gradient_invariants():
    inp = tiny(counts=(3, 5))
    p = oracle_problem(inp)
    do = to_np(inp.do)
    dQ, dK, dV, dKb, dVb = A.backward(p, do)
    w = inp.workload
    ao, ko = inp.anchor_off.tolist(), inp.key_off.tolist()
    for s in range(len(w.seq_lens)):
        rows = slice(w.block * ao[s], w.block * ao[s + 1])
        for g in range(w.n_kv_heads):
            # each softmax row of dS sums to zero, so the key gradients of a kv head cancel
            tot = dK[ko[s]:ko[s + 1], g].sum(0) + dKb[rows, g].sum(0)
            assert np.allclose(tot, 0, atol=1e-12)
            # each softmax row sums to one, so sum_j dV_j = sum over the group's rows of dO
            heads = range(g * w.group, (g + 1) * w.group)
            want = sum(do[rows, h].sum(0) for h in heads)
            got = dV[ko[s]:ko[s + 1], g].sum(0) + dVb[rows, g].sum(0)
            assert np.allclose(got, want, atol=1e-12)


def test_restricted_backward_sums_to_full():
    inp = tiny(counts=(3, 4))
    p = oracle_problem(inp)
    do = to_np(inp.do)
    full = A.backward(p, do)
    part_a = A.backward(p, do, blocks=[0, 2, 4, 6])
    part_b = A.backward(p, do, blocks=[1, 3, 5])
    for f, x, y in zip(full, part_a, part_b):
        np.testing.assert_allclose(x + y, f, atol=1e-13)
