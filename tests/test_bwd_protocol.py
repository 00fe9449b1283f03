"""The one-pass tensor-core backward's barrier protocol, simulated on the CPU.

`bwd_tc_kernel` (split_kv_lse_splitkv_b200/csrc/bwd_tc.cu) coordinates five roles through mbarriers: the TMA
producer, two MMA issuers (A: S^T, dV, dK; B: dP^T, dQ^T), eight elementwise warps and eight dQ warps. This
test restates that protocol (the barriers, their arrival counts, every wait with its phase parity, every
arrival or MMA commit, in each role's program order) and runs it under many random interleavings with the
mbarrier semantics (a phase completes when its count of arrivals is reached; a parity wait succeeds once the
phase of that parity has completed). MMAs are taken to complete when issued, so the check is about order:
no interleaving deadlocks, and no buffer (the Q_b/dO_b slots, the S/P^T and dP^T TMEM buffers, the dQ^T
TMEM buffer, the shared-memory dS^T buffers) is rewritten before its last reader has run. A protocol change
in the kernel goes through this model first; the planted mistakes below show that the checks catch the
errors they are for.
"""
from __future__ import annotations

import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count
        if self.pending == self.count:
            self.pending, self.phase = 0, self.phase + 1

    def done(self, parity):
        return (self.phase & 1) != parity


def simulate(n_pairs, steps, seed, n_elem=8, n_dq=8, mutate=None):
    """Runs every role to completion in a random order; returns the event log. `mutate` plants a mistake."""
    rnd = random.Random(seed)
    U = n_pairs * steps
    bars = {"kv_full": Bar(1), "dp_read": Bar(n_elem), "dq_full": Bar(1), "dq_free": Bar(n_dq),
            "acc_done": Bar(2), "epi_staged": Bar(n_elem)}
    for b in range(2):
        bars[f"qd_full{b}"] = Bar(1)
        bars[f"qd_empty{b}"] = Bar(2)
        bars[f"s_full{b}"] = Bar(2)
        bars[f"p_full{b}"] = Bar(n_elem)
    log = []

    def wait(name, parity):
        return ("wait", name, parity)

    def load():
        log.append(("kv",))
        bars["kv_full"].arrive()
        for p in range(n_pairs):
            yield wait(f"qd_empty{p & 1}", ((p >> 1) & 1) ^ 1)
            log.append(("load", p))
            bars[f"qd_full{p & 1}"].arrive()

    def issuer(is_a):
        yield wait("kv_full", 0)

        def first(u):
            p, h = divmod(u, steps)
            if h == 0:
                yield wait(f"qd_full{p & 1}", (p >> 1) & 1)
            if not is_a and u >= 1 and mutate != "no_dp_read_wait":
                yield wait("dp_read", (u - 1) & 1)
            log.append(("A1" if is_a else "B1", u))          # S^T(u) / dP^T(u)
            bars[f"s_full{u & 1}"].arrive()
            if not is_a and h == steps - 1:
                bars[f"qd_empty{p & 1}"].arrive()             # dO_b read for the last time

        def second(u):
            p, h = divmod(u, steps)
            yield wait(f"p_full{u & 1}", (u >> 1) & 1)
            if is_a:
                log.append(("A2", u))                         # dV(u), dK(u)
                if h == steps - 1:
                    bars[f"qd_empty{p & 1}"].arrive()         # Q_b / dO_b read for the last time
            else:
                if u >= 1 and mutate != "no_dq_free_wait":
                    yield wait("dq_free", (u - 1) & 1)
                log.append(("B2", u))                         # dQ^T(u)
                bars["dq_full"].arrive()

        for u in range(U):
            yield from first(u)
            if u >= 1:
                yield from second(u - 1)
        if U:
            yield from second(U - 1)
            bars["acc_done"].arrive()

    def elementwise(w):
        for u in range(U):
            p = u // steps
            yield wait(f"s_full{u & 1}", (u >> 1) & 1)
            yield wait(f"qd_full{p & 1}", (p >> 1) & 1)
            log.append(("Er", u, w))                          # S^T(u), dP^T(u) into registers
            bars["dp_read"].arrive()
            log.append(("Ew", u, w))                          # P^T(u) into TMEM, dS^T(u) into shared memory
            bars[f"p_full{u & 1}"].arrive()
        if U:
            yield wait("acc_done", 0)
        bars["epi_staged"].arrive()
        yield wait("epi_staged", 0)

    def dq_warp(w):
        for u in range(U):
            yield wait("dq_full", u & 1)
            log.append(("D", u, w))                           # dQ^T(u) out of TMEM
            bars["dq_free"].arrive()

    roles = [load(), issuer(True), issuer(False)] + [elementwise(w) for w in range(n_elem)] + \
        [dq_warp(w) for w in range(n_dq)]
    pending = [None] * len(roles)
    alive = set(range(len(roles)))
    while alive:
        ready = [i for i in alive if pending[i] is None or bars[pending[i][1]].done(pending[i][2])]
        if not ready:
            raise RuntimeError("deadlock: " + ", ".join(f"{pending[i][1]}/{pending[i][2]}" for i in sorted(alive)))
        i = rnd.choice(ready)
        try:
            pending[i] = next(roles[i])
        except StopIteration:
            alive.discard(i)
    return log


def check_order(log, n_pairs, steps, n_elem=8, n_dq=8):
    pos = {e: k for k, e in enumerate(log)}
    U = n_pairs * steps
    for p in range(2, n_pairs):
        last = (p - 2) * steps + steps - 1
        assert pos[("load", p)] > pos[("A2", last)], f"Q_b/dO_b slot reloaded before dV/dK read pair {p - 2}"
        assert pos[("load", p)] > pos[("B1", last)], f"dO_b slot reloaded before dP^T read pair {p - 2}"
    for u in range(U):
        for w in range(n_elem):
            assert pos[("Er", u, w)] > pos[("A1", u)] and pos[("Er", u, w)] > pos[("B1", u)], f"step {u} read early"
            if u >= 2:
                assert pos[("Ew", u, w)] > pos[("A2", u - 2)], f"dS^T buffer of step {u - 2} rewritten before dK"
                assert pos[("Ew", u, w)] > pos[("B2", u - 2)], f"dS^T buffer of step {u - 2} rewritten before dQ^T"
        assert all(pos[("A2", u)] > pos[("Ew", u, w)] for w in range(n_elem)), f"dV/dK({u}) before P^T/dS^T"
        assert all(pos[("B2", u)] > pos[("Ew", u, w)] for w in range(n_elem)), f"dQ^T({u}) before dS^T"
        if u >= 1:
            assert all(pos[("B1", u)] > pos[("Er", u - 1, w)] for w in range(n_elem)), f"dP buffer of step {u - 1}"
            assert all(pos[("B2", u)] > pos[("D", u - 1, w)] for w in range(n_dq)), f"dQ^T buffer of step {u - 1}"
        if u >= 2:
            assert pos[("A1", u)] > pos[("A2", u - 2)], f"S/P^T buffer of step {u - 2}"
        assert all(pos[("D", u, w)] > pos[("B2", u)] for w in range(n_dq)), f"dQ^T({u}) read early"


@pytest.mark.parametrize("n_pairs", [0, 1, 2, 3, 6])
@pytest.mark.parametrize("steps", [1, 2])
def test_protocol_has_no_deadlock_and_keeps_buffer_order(n_pairs, steps):
    for seed in range(150):
        check_order(simulate(n_pairs, steps, seed), n_pairs, steps)


@pytest.mark.parametrize("mutate, expect", [("no_dq_free_wait", "dQ^T buffer|deadlock"),
                                            ("no_dp_read_wait", "dP buffer|deadlock")])
def test_planted_protocol_mistakes_are_caught(mutate, expect):
    # Without B's wait for the dQ warps (or for the elementwise warps' dP^T reads), some interleaving
    # overwrites a TMEM buffer before its reader ran, or a barrier runs two phases ahead of its waiters
    # (whose parity wait then never succeeds).
    with pytest.raises((AssertionError, RuntimeError), match=expect):
        for seed in range(300):
            check_order(simulate(4, 2, seed, mutate=mutate), 4, 2)


def test_planted_count_mistake_deadlocks():
    # A wrong arrival count (the Q_b/dO_b slot released by one issuer only) is a deadlock or an early reuse.
    def run():
        for seed in range(50):
            log = simulate_with_counts(seed)
            check_order(log, 4, 2)

    def simulate_with_counts(seed):
        orig = Bar.__init__

        def patched(self, count):
            orig(self, 3 if count == 2 else count)  # every two-arrival barrier now waits for three
        Bar.__init__ = patched
        try:
            return simulate(4, 2, seed)
        finally:
            Bar.__init__ = orig

    with pytest.raises((RuntimeError, AssertionError)):
        run()
