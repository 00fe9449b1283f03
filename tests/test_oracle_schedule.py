"""Pins of the integer cost / LPT oracle.

* costs: brute-force mask enumeration equals the closed form on random small
  cases (ragged tail chunks, anchors on tile edges), plus a hand-worked example;
* LPT: a hand-worked plan; the textbook worst case of Graham's analysis
  (m = 2, costs 3,3,2,2,2: LPT 7, optimum 6); exhaustive optimum for m <= 3 and
  <= 10 items with LPT <= (4/3 - 1/(3m)) OPT; every item placed exactly once;
  queues in assignment order.
"""
import numpy as np
import pytest

from oracle import schedule as Sch
from tests._util import read_golden


def test_cost_worked_example():
    g = read_golden("cost_worked_example.txt")
    for fn in (Sch.costs_bruteforce, Sch.costs_closed_form):
        kw = dict(group=g["group"]) if fn is Sch.costs_bruteforce else {}
        ids, costs, chunk_costs = fn([g["anchors"]], [g["seq_len"]], g["chunk"], g["key_tile"],
                                     g["n_kv_heads"], **kw)
        assert ids.tolist() == g["item_ids"]
        assert costs.tolist() == g["item_costs"]
        assert chunk_costs.tolist() == g["chunk_costs"]


@pytest.mark.parametrize("seed", range(12))
def test_cost_bruteforce_equals_closed_form(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 4))
    tk = int(rng.choice([8, 16, 32]))
    chunk = tk * int(rng.integers(1, 5))
    hkv = int(rng.integers(1, 3))
    seq, anchors = [], []
    for _ in range(B):
        S = int(rng.integers(20, 300))
        n = int(rng.integers(0, min(6, S - 16) + 1))
        a = sorted(rng.choice(np.arange(16, S), size=n, replace=False).tolist())
        if n and rng.random() < 0.5:  # put one anchor exactly on a tile / chunk edge
            edge = (int(rng.integers(1, max(2, S // tk))) * tk)
            if 16 <= edge < S and edge not in a:
                a = sorted(a[:-1] + [edge])
        seq.append(S)
        anchors.append(a)
    bf = Sch.costs_bruteforce(anchors, seq, chunk, tk, hkv, group=2, block=16)
    cf = Sch.costs_closed_form(anchors, seq, chunk, tk, hkv)
    for x, y in zip(bf, cf):
        assert x.tolist() == y.tolist()
    # every visible context pair lies in a counted tile: tiles * Tk >= visible keys per (block, head)
    layout, total = Sch.item_layout([len(a) for a in anchors], seq, chunk, hkv)
    assert all(i < total for i in bf[0].tolist())
    assert int(bf[1].sum()) * tk >= hkv * sum(sum(a) for a in anchors)


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("pack", [2, 3, 4])
def test_multi_block_tile_costs(seed, pack):
    # Query tiles of `pack` blocks: brute-force mask enumeration equals the closed form, and a tile's
    # cost is the largest of its blocks' one-block costs (their visible key ranges are nested prefixes).
    rng = np.random.default_rng(1000 + seed)
    tk = int(rng.choice([8, 16, 32]))
    chunk = tk * int(rng.integers(1, 5))
    hkv = int(rng.integers(1, 3))
    seq, anchors = [], []
    for _ in range(int(rng.integers(1, 4))):
        S = int(rng.integers(20, 300))
        n = int(rng.integers(0, min(7, S - 16) + 1))
        seq.append(S)
        anchors.append(sorted(rng.choice(np.arange(16, S), size=n, replace=False).tolist()))
    bf = Sch.costs_bruteforce(anchors, seq, chunk, tk, hkv, group=2, block=16, pack=pack)
    cf = Sch.costs_closed_form(anchors, seq, chunk, tk, hkv, pack=pack)
    for x, y in zip(bf, cf):
        assert x.tolist() == y.tolist()
    one = Sch.costs_closed_form(anchors, seq, chunk, tk, hkv)
    one_cost = dict(zip(one[0].tolist(), one[1].tolist()))
    lay1, _ = Sch.item_layout([len(a) for a in anchors], seq, chunk, hkv)
    layp, _ = Sch.item_layout([len(a) for a in anchors], seq, chunk, hkv, pack)
    got = dict(zip(cf[0].tolist(), cf[1].tolist()))
    for s, a in enumerate(anchors):
        (b1, nc, nb), (bp, _, nt) = lay1[s], layp[s]
        assert nt == -(-len(a) // pack)
        for c in range(nc):
            for g in range(hkv):
                for t in range(nt):
                    members = range(t * pack, min((t + 1) * pack, nb))
                    want = max(one_cost.get(b1 + (c * hkv + g) * nb + b, 0) for b in members)
                    assert got.get(bp + (c * hkv + g) * nt + t, 0) == want
    assert cf[2].tolist() != [] or not seq  # chunk costs present for every chunk


def test_chunk_runs_worked_example():
    # Runs of chunks, worked by hand: S = 640, C = Tk = 128 (five chunks), runs of L = 2 chunks (three
    # runs: keys [0,256), [256,512), [512,640)), one kv head, one block with anchor 300.
    #   run 0 sees keys [0,256): 2 tiles; run 1 sees [256,300): 1 tile; run 2 sees none (dropped);
    #   chunks 0, 1, 2 each hold one visible tile ([0,128), [128,256), [256,300)); chunks 3, 4 none.
    for fn, kw in ((Sch.costs_bruteforce, dict(group=1)), (Sch.costs_closed_form, {})):
        ids, costs, chunk_costs = fn([[300]], [640], 128, 128, 1, runs=2, **kw)
        assert ids.tolist() == [0, 1]
        assert costs.tolist() == [2, 1]
        assert chunk_costs.tolist() == [1, 1, 1, 0, 0]
    layout, total = Sch.item_layout([1], [640], 128, 1, runs=2)
    assert layout == [(0, 3, 1)] and total == 3


@pytest.mark.parametrize("seed", range(10))
@pytest.mark.parametrize("runs", [2, 3, 8])
@pytest.mark.parametrize("pack", [1, 2])
def test_chunk_run_costs(seed, runs, pack):
    # Runs of L chunks: brute-force mask enumeration equals the closed form; the chunk costs do not
    # depend on L; every item tile lies in exactly one chunk (item costs and chunk costs add up to the
    # same total); and a run's cost is the sum of its chunks' one-chunk item costs (a run's visible keys
    # are the union of its chunks' visible keys, tile-aligned).
    rng = np.random.default_rng(2000 + seed)
    tk = int(rng.choice([8, 16, 32]))
    chunk = tk * int(rng.integers(1, 9))  # up to 8 cost tiles per chunk (256-key tiles on 2048-key chunks)
    hkv = int(rng.integers(1, 3))
    seq, anchors = [], []
    for _ in range(int(rng.integers(1, 4))):
        S = int(rng.integers(20, 40 * chunk // tk + 300))
        n = int(rng.integers(0, min(6, S - 16) + 1))
        seq.append(S)
        anchors.append(sorted(rng.choice(np.arange(16, S), size=n, replace=False).tolist()))
    bf = Sch.costs_bruteforce(anchors, seq, chunk, tk, hkv, group=2, block=16, pack=pack, runs=runs)
    cf = Sch.costs_closed_form(anchors, seq, chunk, tk, hkv, pack=pack, runs=runs)
    for x, y in zip(bf, cf):
        assert x.tolist() == y.tolist()
    one = Sch.costs_closed_form(anchors, seq, chunk, tk, hkv, pack=pack)
    assert cf[2].tolist() == one[2].tolist()
    assert int(cf[1].sum()) == int(cf[2].sum())
    one_cost = dict(zip(one[0].tolist(), one[1].tolist()))
    lay1, _ = Sch.item_layout([len(a) for a in anchors], seq, chunk, hkv, pack)
    layr, _ = Sch.item_layout([len(a) for a in anchors], seq, chunk, hkv, pack, runs)
    got = dict(zip(cf[0].tolist(), cf[1].tolist()))
    for s in range(len(seq)):
        (b1, nc, nt), (br, nr, _) = lay1[s], layr[s]
        assert nr == -(-nc // runs)
        for r in range(nr):
            for g in range(hkv):
                for t in range(nt):
                    want = sum(one_cost.get(b1 + (c * hkv + g) * nt + t, 0)
                               for c in range(r * runs, min((r + 1) * runs, nc)))
                    assert got.get(br + (r * hkv + g) * nt + t, 0) == want


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("overhead", [1, 3])
def test_item_overhead_costs(seed, overhead):
    # The per-item constant: brute force equals the closed form; every visible item (and only those)
    # costs exactly kappa more than without it; the chunk costs do not change.
    rng = np.random.default_rng(3000 + seed)
    tk = int(rng.choice([8, 16]))
    chunk = tk * int(rng.integers(1, 4))
    seq, anchors = [], []
    for _ in range(int(rng.integers(1, 3))):
        S = int(rng.integers(30, 250))
        n = int(rng.integers(1, min(5, S - 16) + 1))
        seq.append(S)
        anchors.append(sorted(rng.choice(np.arange(16, S), size=n, replace=False).tolist()))
    bf = Sch.costs_bruteforce(anchors, seq, chunk, tk, 2, group=2, block=16, pack=2, runs=2, overhead=overhead)
    cf = Sch.costs_closed_form(anchors, seq, chunk, tk, 2, pack=2, runs=2, overhead=overhead)
    base = Sch.costs_closed_form(anchors, seq, chunk, tk, 2, pack=2, runs=2)
    for x, y in zip(bf, cf):
        assert x.tolist() == y.tolist()
    assert cf[0].tolist() == base[0].tolist()
    assert (cf[1] - base[1]).tolist() == [overhead] * len(base[1])
    assert cf[2].tolist() == base[2].tolist()


def test_lpt_worked_example():
    g = read_golden("lpt_worked_example.txt")
    iw, qo, qi, load = Sch.lpt(g["costs"], g["n_workers"])
    assert iw.tolist() == g["item_worker"]
    assert qo.tolist() == g["queue_off"]
    assert qi.tolist() == g["queue_items"]
    assert load.tolist() == g["load"]


def test_lpt_graham_worst_case():
    costs = [3, 3, 2, 2, 2]
    _, _, _, load = Sch.lpt(costs, 2)
    assert Sch.makespan(load) == 7
    assert Sch.optimal_makespan(costs, 2) == 6
    assert 7 <= (4 / 3 - 1 / 6) * 6 + 1e-12


@pytest.mark.parametrize("seed", range(40))
def test_lpt_within_graham_bound_of_exhaustive_optimum(seed):
    rng = np.random.default_rng(100 + seed)
    m = int(rng.integers(1, 4))
    n = int(rng.integers(0, 11 if m < 3 else 10))
    costs = rng.integers(1, 9, size=n).tolist()
    iw, qo, qi, load = Sch.lpt(costs, m)
    opt = Sch.optimal_makespan(costs, m)
    assert Sch.makespan(load) <= (4 / 3 - 1 / (3 * m)) * opt + 1e-9
    # every item exactly once; queues consistent with item_worker; loads add up
    assert sorted(qi.tolist()) == list(range(n))
    for w in range(m):
        q = qi[qo[w]:qo[w + 1]].tolist()
        assert all(iw[i] == w for i in q)
        assert sum(costs[i] for i in q) == load[w]
        # assignment order: non-increasing cost, ascending index among equal costs
        keys = [(-costs[i], i) for i in q]
        assert keys == sorted(keys)


def test_lpt_tie_breaks_prefer_lower_worker_and_lower_index():
    iw, qo, qi, load = Sch.lpt([1, 1, 1, 1], 3)
    assert iw.tolist() == [0, 1, 2, 0]
    assert load.tolist() == [2, 1, 1]


def test_naive_split_contiguous_equal_counts():
    costs = [5, 1, 1, 1, 1, 1, 1]
    iw, qo, qi, load = Sch.naive_split(costs, 3)
    assert qo.tolist() == [0, 2, 4, 7]
    assert load.tolist() == [6, 2, 3]
    assert Sch.imbalance(load) == pytest.approx(6 / (11 / 3) - 1)
