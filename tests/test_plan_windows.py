"""The run-window decomposition behind the device planner, checked on the CPU against the heap LPT.

`plan_runs_kernel` (split_kv_lse_splitkv_b200/csrc/plan.cu) does not place items one at a time. It takes
each run of equal-cost items as a whole: with cost w, worker i offers loads L_i, L_i + w, L_i + 2w, ...;
cutting the load axis into windows of width w from the minimum load V0 gives worker i a first window
r_i = (L_i - V0) // w and an offset o_i = (L_i - V0) % w, so every window lists its workers in the same
(offset, worker) order q. Windows below R = max r_i hold only the workers that reached them ("catch-up");
from R on, every window holds all m workers in q order. The run's n items take the first n ranks.

This file restates that decomposition in plain Python (no kernel, no oracle code) and requires it to give
the oracle's greedy (longest processing time first: cost descending, index ascending, least (load,
worker)) for every item, queue and load, over worker counts and cost mixes like the workloads'.
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import schedule as OS


def windows_plan(costs, m):
    """Items' workers and queues, run by run, by the window decomposition."""
    costs = list(costs)
    order = sorted(range(len(costs)), key=lambda k: (-costs[k], k))
    load = [0] * m
    queues = [[] for _ in range(m)]
    worker_of = [0] * len(costs)
    pos = 0
    while pos < len(order):
        w = costs[order[pos]]
        run = []
        while pos < len(order) and costs[order[pos]] == w:
            run.append(order[pos])
            pos += 1
        n = len(run)
        v0 = min(load)
        r = [(x - v0) // w for x in load]
        o = [(x - v0) % w for x in load]
        q = sorted(range(m), key=lambda i: (o[i], i))        # the order inside every window
        R = max(r)
        picks = []                                           # (worker) in rank order
        for win in range(R):                                 # catch-up windows
            picks += [i for i in q if r[i] <= win]
            if len(picks) >= n:
                break
        win = R
        while len(picks) < n:                                # steady windows: all workers, q order
            picks += q
            win += 1
        for k, i in zip(run, picks[:n]):
            worker_of[k] = i
            queues[i].append(k)
            load[i] += w
    queue_off = np.concatenate([[0], np.cumsum([len(x) for x in queues])]).astype(np.int64)
    queue_items = [k for x in queues for k in x]
    return worker_of, queue_off.tolist(), queue_items, load


def check(costs, m):
    iw, qo, qi, ld = OS.lpt(list(costs), m)
    got = windows_plan(costs, m)
    assert got[0] == iw.tolist()
    assert got[1] == qo.tolist()
    assert got[2] == qi.tolist()
    assert got[3] == ld.tolist()


@pytest.mark.parametrize("m", [1, 2, 31, 33, 64, 65, 100, 148, 224, 256, 300])
@pytest.mark.parametrize("seed", range(3))
def test_windows_equal_the_greedy_on_random_costs(m, seed):
    # Every bucket 1..64 present, skewed towards small costs (as in the planner's GPU test), ties everywhere.
    rng = np.random.default_rng(100 * m + seed)
    n = int(rng.integers(64, 1500))
    costs = np.minimum(64, rng.geometric(0.08, size=n))
    costs[:64] = np.arange(1, 65)
    rng.shuffle(costs)
    check(costs.tolist(), m)


@pytest.mark.parametrize("name,tk,runs,pack", [("drafter_s32k", 128, 6, 1), ("long_s128k", 256, 8, 1),
                                               ("long_s128k", 128, 4, 1), ("skewed_s256k", 256, 8, 2)])
def test_windows_equal_the_greedy_on_workload_costs(name, tk, runs, pack):
    # The full-size workloads' own item costs (closed form of the oracle) on one queue per SM.
    import workloads as W
    from tests._util import anchors_per_sample
    inp = W.make_inputs(W.get(name))
    w = inp.workload
    _, costs, _ = OS.costs_closed_form(anchors_per_sample(inp), w.seq_lens, w.chunk, tk, w.n_kv_heads, pack=pack,
                                       runs=runs)
    check(costs.tolist(), 148)


def test_catch_up_windows_are_bounded():
    # The device sizes run w's catch-up list by m * (W // w): every load stays within the largest cost W of
    # the minimum, so r_i <= W // w. Checked along the greedy on adversarial mixes (one huge item first).
    rng = np.random.default_rng(7)
    for _ in range(40):
        m = int(rng.integers(1, 40))
        W_ = int(rng.integers(1, 65))
        costs = rng.integers(1, W_ + 1, size=int(rng.integers(1, 400))).tolist()
        costs[0] = W_
        load = [0] * m
        for k in sorted(range(len(costs)), key=lambda k: (-costs[k], k)):
            w = costs[k]
            assert max(load) - min(load) <= W_
            assert max((x - min(load)) // w for x in load) <= W_ // w
            i = min(range(m), key=lambda j: (load[j], j))
            load[i] += w
