"""Parity of the CUDA path (through the C ABI) with the float64 CPU oracle on seeded inputs.

Costs and plans bit for bit; partials, O, LSE and gradients within the tolerances in tests/_gpu.py.
Small cases compare every element and span several key tiles, chunks, ragged tails and queues;
the full-size workloads compare the integer outputs completely and sampled rows of the floats.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from tests._gpu import (assert_close, check_cost_and_plan, check_partials, counts_of, run_forward)
from tests._util import oracle_problem, to_np

pytestmark = pytest.mark.gpu

SIMT = 1


def small(name, base, seq_lens, counts, chunk=None, seed=11, **kw):
    # Items over one chunk, costs in 128-key tiles, unless a test asks otherwise (the full-size workloads
    # use runs of chunks, long_s128k and skewed_s256k a coarser cost tile).
    kw.setdefault("chunks_per_item", 1)
    kw.setdefault("key_tile", 128)
    return W.make_inputs(W.scaled(W.get(base), name, seq_lens, counts, chunk=chunk, seed=seed, **kw))


def full_check(inp, n_workers, flags=0, partials=True, magnitude_scaled=False):
    skv, dev, anchors, o, lse = run_forward(inp, n_workers=n_workers, flags=flags)
    skv.check_status()
    ids, _ = check_cost_and_plan(skv, inp)
    if partials:
        check_partials(skv, inp, ids, magnitude_scaled)
    O, L = OA.forward(oracle_problem(inp))
    dt = inp.workload.dtype
    assert_close("O", to_np(o), O, dt, magnitude_scaled)
    assert_close("LSE", to_np(lse), L, dt)
    return skv, dev, anchors, o, lse


def test_tiny_f32_workload():
    # 1 q / 1 kv head, d = 64, S = 1024, 4 anchors, chunk 128, 4 workers: the whole workload.
    full_check(W.make_inputs(W.get("tiny_f32")), n_workers=4)


@pytest.mark.parametrize("hq,hkv,P", [(24, 8, 1), (24, 8, 2), (48, 8, 1)])
def test_group_sizes_not_powers_of_two(hq, hkv, P):
    # G = 3 (48-row blocks, alone or two to a tile) and G = 6 (96 rows): rows past the block's in the
    # 128-row MMA tile stay masked.
    inp = small("groups_odd", "skewed_s256k", [4096], [9], chunk=2048, n_q_heads=hq, n_kv_heads=hkv, blocks_per_item=P)
    full_check(inp, n_workers=5)


@pytest.mark.parametrize("flags", [0, SIMT])
@pytest.mark.parametrize("n_workers", [3, 148])
def test_drafter_shape_small(flags, n_workers):
    # GQA 8 (one 128-row query tile per item), S = 5000: ragged last chunk and ragged key tiles.
    inp = small("drafter_small", "drafter_s32k", [5000], [7], chunk=1024)
    full_check(inp, n_workers, flags)


@pytest.mark.parametrize("flags", [0, SIMT])
def test_score_jumps_inside_items(flags):
    # Keys with 12x the norm make a row's running max jump far past the lazy-rescale threshold: in
    # an item's first tile, in the first and in the second half of later tiles. The softmax must
    # move its reference max there (rescaling O, the row sum and the part of P already written).
    inp = small("jumps", "drafter_s32k", [3000], [6], chunk=1024, seed=13)
    for pos in (5, 2 * 128 + 10, 3 * 128 + 100, 1024 + 5 * 128 + 70, 2048 + 4 * 128 + 88):
        inp.k[pos] *= 12
    full_check(inp, n_workers=7, flags=flags, magnitude_scaled=True)


@pytest.mark.parametrize("full_tiles", [False, True])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 4), (4, 4)])
def test_other_group_sizes(hq, hkv, full_tiles):
    # G = 4, 2, 1: 64-, 32- and 16-row blocks, alone in the 128-row MMA tile or 128/(16G) of them
    # sharing it (9 blocks: the sample's last tile is partly empty).
    P = 128 // (16 * (hq // hkv)) if full_tiles else 1
    inp = small("groups", "skewed_s256k", [4096], [9], chunk=2048, n_q_heads=hq, n_kv_heads=hkv, blocks_per_item=P)
    full_check(inp, n_workers=5)


@pytest.mark.parametrize("flags", [0, SIMT])
def test_multi_block_tiles_batch(flags):
    # Two blocks per query tile across three samples with 3, 1 and 4 blocks (odd counts leave half-empty
    # tiles at sample ends, where the next sample's rows follow in memory) and ragged chunks.
    inp = small("packs", "skewed_s256k", [3000, 700, 5000], [3, 1, 4], chunk=1024, blocks_per_item=2)
    full_check(inp, n_workers=6, flags=flags)


# ------------------------------------------------------------------ pairs of SMs (256-row items)
@pytest.mark.parametrize("flags", [0, SIMT])
@pytest.mark.parametrize("n_workers", [3, None])
def test_pair_kernel_drafter_shape(flags, n_workers):
    # Two 128-row blocks (G = 8) per 256-row item, one per SM of a two-CTA cluster; 7 blocks leave the
    # last tile with one block (the peer CTA's rows are empty). None: the co-resident pair count.
    inp = small("drafter_pair", "drafter_s32k", [5000], [7], chunk=1024, blocks_per_item=2)
    full_check(inp, n_workers, flags)


@pytest.mark.parametrize("hq,hkv,P", [(32, 8, 4), (8, 4, 8)])
def test_pair_kernel_other_group_sizes(hq, hkv, P):
    # G = 4 (two 64-row blocks per SM) and G = 2 (four 32-row blocks per SM); 9 blocks: ragged last tile.
    inp = small("pair_groups", "skewed_s256k", [4096], [9], chunk=2048, n_q_heads=hq, n_kv_heads=hkv,
                blocks_per_item=P)
    full_check(inp, n_workers=5)


def test_pair_kernel_batch_edges_and_jumps():
    # Three samples (3, 1 and 4 blocks, ragged chunks), anchors on tile and chunk boundaries, and keys of
    # 12x the norm that move the running max inside items.
    w = W.scaled(W.get("drafter_s32k"), "pair_batch", [3000, 700, 5000], [3, 1, 4], chunk=1024, seed=13,
                 blocks_per_item=2)
    inp = W.make_inputs(w)
    inp.anchors = torch.tensor([127, 128, 2999, 16, 1023, 1024, 1025, 4999], dtype=torch.int32)
    for pos in (5, 2 * 128 + 10, 3700 + 1024 + 5 * 128 + 70):
        inp.k[pos] *= 12
    full_check(inp, n_workers=4, magnitude_scaled=True)


def test_pair_kernel_wait_limit_returns_a_status():
    from split_kv_lse_splitkv_b200 import DEV_TIMEOUT, FWD_TEST_STARVE
    inp = small("pair_starve", "drafter_s32k", [5000], [7], chunk=1024, blocks_per_item=2)
    skv, dev, anchors, o_ref, lse_ref = run_forward(inp, n_workers=4)
    skv.check_status()
    skv.plan(anchors)
    skv.attn_fwd(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], anchors, flags=FWD_TEST_STARVE)
    torch.cuda.synchronize()
    assert skv.status_value() & DEV_TIMEOUT, skv.status_value()
    skv.status.zero_()
    o, lse = skv.forward(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], anchors)
    torch.cuda.synchronize()
    skv.check_status()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


# ------------------------------------------------------------------ runs of chunks per item
@pytest.mark.parametrize("flags", [0, SIMT])
@pytest.mark.parametrize("runs,P", [(2, 1), (3, 1), (2, 2), (3, 2)])
def test_runs_of_chunks(flags, runs, P):
    # Items over runs of 2 or 3 chunks of 512 keys (ragged last run, S = 5000), one SM (P = 1) or a pair
    # of SMs (P = 2) per worker: one partial per run, chunk costs per chunk, and O/LSE as always.
    inp = small("runs", "drafter_s32k", [5000], [7], chunk=512, blocks_per_item=P, chunks_per_item=runs)
    full_check(inp, n_workers=5, flags=flags)


def test_item_overhead_plan():
    # The per-item constant of the cost: costs and the LPT plan equal the oracle's bit for bit, and the
    # forward is unchanged by it.
    inp = small("overhead", "drafter_s32k", [5000, 3000], [7, 4], chunk=512, chunks_per_item=2, item_overhead=3)
    full_check(inp, n_workers=9)


def test_runs_of_chunks_batch_and_groups():
    # Three samples, G = 4 with two blocks per 128-row tile, runs of 2 chunks of 1024 keys.
    inp = small("runs_batch", "skewed_s256k", [3000, 700, 5000], [3, 1, 4], chunk=1024, blocks_per_item=2,
                chunks_per_item=2)
    full_check(inp, n_workers=6)


def test_long_runs_coarse_cost_tile():
    # Runs of 16 chunks whose cost counts 512-key tiles (skewed_s256k's setting), two blocks per 128-row
    # tile: items of up to 16384 keys in one pass of the online softmax, ragged last runs, two samples.
    inp = small("long_runs", "skewed_s256k", [40000, 9000], [5, 2], chunk=1024, blocks_per_item=2,
                chunks_per_item=16, key_tile=512)
    full_check(inp, n_workers=6)


def test_anchor_edges():
    # Anchors on key-tile and chunk boundaries, the smallest and the largest allowed anchor.
    w = W.scaled(W.get("drafter_s32k"), "edges", [2048], [8], chunk=1024)
    inp = W.make_inputs(w)
    inp.anchors = torch.tensor([16, 127, 128, 129, 1023, 1024, 1025, 2047], dtype=torch.int32)
    full_check(inp, n_workers=4)


def test_batch_and_single_worker():
    inp = small("batch", "train_4x64k", [3000, 2048, 4096], [2, 3, 4], chunk=1024)
    full_check(inp, n_workers=1)


def test_tensor_core_and_simt_kernels_agree():
    inp = small("agree", "long_s128k", [16384], [12], chunk=2048)
    _, _, _, o_tc, l_tc = run_forward(inp, n_workers=16, flags=0)
    _, _, _, o_si, l_si = run_forward(inp, n_workers=16, flags=SIMT)
    assert_close("O tc vs simt", to_np(o_tc), to_np(o_si), "bf16")
    assert_close("LSE tc vs simt", to_np(l_tc), to_np(l_si), "bf16")


def backward_check(inp, n_workers=4):
    skv, dev, anchors, o, lse = run_forward(inp, n_workers=n_workers)
    do = inp.do.to("cuda")
    grads = skv.backward(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], o, lse, do, anchors)
    torch.cuda.synchronize()
    skv.check_status()
    p = oracle_problem(inp)
    ref = OA.backward(p, to_np(inp.do))
    for name, g, r in zip(("dQ", "dK", "dV", "dKb", "dVb"), grads, ref):
        assert_close(name, to_np(g), r, inp.workload.dtype)


def test_backward_bf16_batch():
    backward_check(small("bwd", "train_4x64k", [3000, 2048, 4096], [2, 3, 4], chunk=1024))


@pytest.mark.parametrize("full_tiles", [False, True])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 4), (4, 4)])
def test_backward_other_group_sizes(hq, hkv, full_tiles):
    # G = 4, 2, 1: 64-, 32- and 16-row blocks, one per query tile or sharing it; ragged key tiles at
    # both sample ends.
    P = 128 // (16 * (hq // hkv)) if full_tiles else 1
    inp = small("bwd_groups", "train_4x64k", [2500, 1300], [3, 2], chunk=1024, n_q_heads=hq, n_kv_heads=hkv,
                blocks_per_item=P)
    backward_check(inp, n_workers=5)


@pytest.mark.parametrize("hq,hkv", [(24, 8), (48, 8)])
def test_backward_group_sizes_not_powers_of_two(hq, hkv):
    # G = 3 (48-row blocks, one step) and G = 6 (96 rows: a second step half inside the block): the dQ
    # reductions walk query rows with a running (query, head) position instead of a compile-time group.
    inp = small("bwd_groups_odd", "train_4x64k", [2500, 1300], [3, 2], chunk=1024, n_q_heads=hq, n_kv_heads=hkv)
    backward_check(inp, n_workers=5)


def test_backward_runs_of_chunks():
    # The forward (whose O and LSE the backward starts from) runs items over 2 chunks of 512 keys; the
    # backward is key-tile stationary whatever the items are.
    backward_check(small("bwd_runs", "train_4x64k", [3000, 2048, 4096], [2, 3, 4], chunk=512, chunks_per_item=2))


def test_backward_f32_tiny():
    w = W.scaled(W.get("tiny_f32"), "bwd_f32", [1024], [4], backward=True)
    backward_check(W.make_inputs(w))


def test_bad_anchors_raise_device_status():
    from split_kv_lse_splitkv_b200 import DEV_ANCHOR_ORDER, DEV_ANCHOR_RANGE
    w = W.scaled(W.get("drafter_s32k"), "bad", [2048], [4], chunk=1024)
    for anchors, bit in (([100, 50, 300, 400], DEV_ANCHOR_ORDER), ([100, 200, 300, 4096], DEV_ANCHOR_RANGE),
                         ([3, 200, 300, 400], DEV_ANCHOR_RANGE)):
        inp = W.make_inputs(w)
        inp.anchors = torch.tensor(anchors, dtype=torch.int32)
        skv, *_ = run_forward(inp, n_workers=4)
        assert skv.status_value() & bit


def test_in_kernel_wait_limit_returns_a_status():
    """The forward's waits are bounded. In test mode the first CTA gets no item and a 20 us limit, so
    every role of it waits, with no copy or MMA issued, until the limit runs out: the kernel must end,
    raise SPLITKV_DEV_TIMEOUT and leave the context usable, so that the next call (status cleared)
    gives exactly what a call without the test mode gives."""
    from split_kv_lse_splitkv_b200 import DEV_TIMEOUT, FWD_TEST_STARVE
    inp = small("starve", "drafter_s32k", [5000], [7], chunk=1024)
    skv, dev, anchors, o_ref, lse_ref = run_forward(inp, n_workers=4)
    skv.check_status()
    skv.plan(anchors)
    skv.attn_fwd(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], anchors, flags=FWD_TEST_STARVE)
    torch.cuda.synchronize()
    assert skv.status_value() & DEV_TIMEOUT, skv.status_value()
    skv.status.zero_()
    o, lse = skv.forward(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], anchors)
    torch.cuda.synchronize()
    skv.check_status()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_planner_rejects_out_of_range_costs():
    from split_kv_lse_splitkv_b200 import DEV_BAD_COST, SplitKV
    skv = SplitKV([4096], [4], 32, 4, 128, chunk=1024, n_workers=8)
    skv.item_cost[:8] = torch.tensor([1, 2, 3, 99, 1, 1, 1, 1], dtype=torch.int32, device="cuda")
    skv.n_items.fill_(8)
    skv.plan_lpt()
    torch.cuda.synchronize()
    assert skv.status_value() & DEV_BAD_COST


@pytest.mark.parametrize("n_workers", [1, 31, 33, 64, 65, 100, 148, 224, 256, 257, 300])
def test_planner_random_costs(n_workers):
    # The run walk (one CTA, a thread per worker, at least four warps) must give the oracle's LPT plan bit
    # for bit for worker counts below, at and above one, two and four warps' worth, the SM count and eight
    # warps. Costs cover every bucket 1..64, skewed towards small ones like the workloads', with a few
    # thousand items so most runs are non-trivial.
    from oracle import schedule as OS
    from split_kv_lse_splitkv_b200 import SplitKV
    skv = SplitKV([262144], [512], 32, 4, 128, chunk=8192, n_workers=n_workers)
    W_ = int(skv.sizes.max_cost)
    n = min(int(skv.sizes.n_items_max), 3000)
    rng = np.random.default_rng(17 + n_workers)
    costs = np.minimum(W_, rng.geometric(0.08, size=n)).astype(np.int32)
    costs[:W_] = np.arange(1, W_ + 1)
    rng.shuffle(costs)
    skv.item_cost[:n] = torch.from_numpy(costs).cuda()
    skv.n_items.fill_(n)
    skv.plan_lpt()
    torch.cuda.synchronize()
    skv.check_status()
    iw, qo, qi, load = OS.lpt(costs.tolist(), n_workers)
    assert skv.item_worker[:n].cpu().numpy().tolist() == iw.tolist()
    assert skv.queue_off.cpu().numpy().tolist() == qo.tolist()
    assert skv.queue_items[:n].cpu().numpy().tolist() == qi.tolist()
    assert skv.load.cpu().numpy().tolist() == load.tolist()


# ------------------------------------------------------------------ full-size workloads
def sampled_blocks(inp, k=4):
    n = int(inp.anchor_off[-1])
    rng = np.random.default_rng(5)
    picks = {0, n - 1, n // 2} | set(rng.integers(0, n, size=max(0, k - 3)).tolist())
    return sorted(picks)


@pytest.mark.parametrize("name", ["drafter_s32k", "long_s128k", "skewed_s256k"])
def test_full_size_forward(name):
    inp = W.make_inputs(W.get(name))
    skv, dev, anchors, o, lse = run_forward(inp)
    skv.check_status()
    check_cost_and_plan(skv, inp)
    blocks = sampled_blocks(inp)
    w = inp.workload
    heads = [0, w.n_q_heads // 2 + 1, w.n_q_heads - 1]
    O, L = OA.forward(oracle_problem(inp), heads=heads, blocks=blocks)
    rows = np.concatenate([np.arange(w.block * j, w.block * (j + 1)) for j in blocks])
    assert_close("O sampled", to_np(o)[rows][:, heads], O[rows][:, heads], w.dtype)
    assert_close("LSE sampled", to_np(lse)[rows][:, heads], L[rows][:, heads], w.dtype)


def test_full_size_training_step():
    inp = W.make_inputs(W.get("train_4x64k"))
    w = inp.workload
    skv, dev, anchors, o, lse = run_forward(inp)
    do = inp.do.to("cuda")
    dq, dk, dv, dkb, dvb = skv.backward(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], o, lse, do, anchors)
    torch.cuda.synchronize()
    skv.check_status()
    check_cost_and_plan(skv, inp)
    p = oracle_problem(inp)
    off, ko = inp.anchor_off.tolist(), inp.key_off.tolist()
    # The last block of each sample is the only one that sees keys [a_{n-2}, a_{n-1}); keys at or
    # beyond its anchor are seen by nobody. Its oracle-only gradients pin those dK/dV rows exactly.
    lasts = [off[s + 1] - 1 for s in range(len(off) - 1)]
    blocks = sorted(set(lasts + [0, off[2]]))
    O, L = OA.forward(p, blocks=blocks)
    ref = OA.backward(p, to_np(inp.do), O=O, LSE=L, blocks=lasts)
    rows = np.concatenate([np.arange(w.block * j, w.block * (j + 1)) for j in blocks])
    assert_close("O sampled", to_np(o)[rows], O[rows], w.dtype)
    assert_close("LSE sampled", to_np(lse)[rows], L[rows], w.dtype)
    last_rows = np.concatenate([np.arange(w.block * j, w.block * (j + 1)) for j in lasts])
    assert_close("dQ sampled", to_np(dq)[last_rows], ref[0][last_rows], w.dtype)
    assert_close("dKb sampled", to_np(dkb)[last_rows], ref[3][last_rows], w.dtype)
    assert_close("dVb sampled", to_np(dvb)[last_rows], ref[4][last_rows], w.dtype)
    anchors_np = inp.anchors.numpy()
    got_k, ref_k, got_v, ref_v = [], [], [], []
    for s in range(len(w.seq_lens)):
        lo = int(anchors_np[off[s + 1] - 2]) if off[s + 1] - off[s] > 1 else 0
        hi = int(anchors_np[off[s + 1] - 1])
        sl = slice(ko[s] + lo, ko[s] + hi)
        got_k.append(to_np(dk)[sl]); ref_k.append(ref[1][sl])
        got_v.append(to_np(dv)[sl]); ref_v.append(ref[2][sl])
        # keys nobody sees
        assert np.all(to_np(dk)[ko[s] + hi:ko[s + 1]] == 0) and np.all(to_np(dv)[ko[s] + hi:ko[s + 1]] == 0)
    assert_close("dK sampled", np.concatenate(got_k), np.concatenate(ref_k), w.dtype)
    assert_close("dV sampled", np.concatenate(got_v), np.concatenate(ref_v), w.dtype)
    # Softmax invariants over every key of each (sample, kv head).
    dkn, dvn, dkbn, dvbn, don = to_np(dk), to_np(dv), to_np(dkb), to_np(dvb), to_np(inp.do)
    for s in range(len(w.seq_lens)):
        r = slice(w.block * off[s], w.block * off[s + 1])
        for g in range(w.n_kv_heads):
            tot_k = dkn[ko[s]:ko[s + 1], g].sum(0) + dkbn[r, g].sum(0)
            mag_k = np.abs(dkn[ko[s]:ko[s + 1], g]).sum(0) + np.abs(dkbn[r, g]).sum(0)
            assert np.all(np.abs(tot_k) <= 1e-3 * mag_k.max() + 1e-6)
            want_v = sum(don[r, h].sum(0) for h in range(g * w.group, (g + 1) * w.group))
            got_v_ = dvn[ko[s]:ko[s + 1], g].sum(0) + dvbn[r, g].sum(0)
            assert np.allclose(got_v_, want_v, rtol=1e-3, atol=1e-2)


# ------------------------------------------------------------------ CUDA graph of the step
@pytest.mark.parametrize("backward", [False, True])
def test_cuda_graph_replay_matches_eager(backward):
    """The step (cost, plan, forward, merge[, backward]) captured once as a CUDA graph and replayed
    on new inputs gives what eager launches give on those inputs (the same bits, dQ to rounding):
    every launch is stream ordered and takes its sizes from the problem, not from device data read
    on the host."""
    from split_kv_lse_splitkv_b200 import SplitKV
    base = "train_4x16k" if backward else "drafter_s32k"
    inp = small("graph", base, [4096, 3072], [6, 4], chunk=1024, seed=21)
    w = inp.workload
    skv = SplitKV(w.seq_lens, counts_of(inp), w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.chunk, w.key_tile,
                  w.scale, w.torch_dtype, n_workers=148, device="cuda", blocks_per_item=w.blocks_per_item,
                  chunks_per_item=w.chunks_per_item)
    names = ("q", "k", "v", "kb", "vb") + (("do",) if backward else ())
    dev = {k: getattr(inp, k).cuda() for k in names}
    anchors = inp.anchors.cuda()
    o = torch.empty(inp.q.shape, dtype=w.torch_dtype, device="cuda")
    lse = torch.empty(inp.q.shape[:2], dtype=torch.float32, device="cuda")
    f = dict(dtype=torch.float32, device="cuda")
    grads = (torch.empty(inp.q.shape, **f), torch.empty(inp.k.shape, **f), torch.empty(inp.v.shape, **f),
             torch.empty(inp.kb.shape, **f), torch.empty(inp.vb.shape, **f))
    stream = torch.cuda.Stream()

    def step():
        skv.forward(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], anchors, o=o, lse=lse, stream=stream)
        if backward:
            skv.backward(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], o, lse, dev["do"], anchors, grads,
                         stream=stream)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
        step()
    torch.cuda.synchronize()
    # New values in the same buffers: the replay must compute from them, not repeat the capture's.
    gen = torch.Generator().manual_seed(5)
    for k in names:
        dev[k].copy_(torch.randn(dev[k].shape, generator=gen).to(dev[k].dtype))
    graph.replay()
    torch.cuda.synchronize()
    skv.check_status()
    got = [o.clone(), lse.clone()] + ([g.clone() for g in grads] if backward else [])
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    ref = [o, lse] + (list(grads) if backward else [])
    for i, (a, b) in enumerate(zip(got, ref)):
        if i == 2:  # dQ: summed over items with float atomics, so the order of the additions varies
            assert torch.allclose(a, b, rtol=1e-5, atol=1e-6 * float(b.abs().max())), "dQ"
        else:
            assert torch.equal(a, b), i


def test_batch_with_an_empty_sample():
    # The middle sample has no anchor: no block, item or self partial of its own, while its keys sit
    # between the other samples' in K and V (their gradients must come out zero).
    inp = small("empty_mid", "train_4x64k", [3000, 2048, 2500], [4, 0, 3], chunk=1024, seed=21)
    full_check(inp, n_workers=5)
    backward_check(inp, n_workers=5)


def test_problem_without_anchors():
    # No anchor at all: empty query tensors (NULL device pointers), no item, an empty plan, zero
    # chunk costs and zero key gradients.
    inp = small("empty_all", "train_4x64k", [2048], [0], chunk=1024, seed=22)
    full_check(inp, n_workers=3)
    backward_check(inp, n_workers=3)
