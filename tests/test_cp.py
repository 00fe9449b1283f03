"""Split-KV context parallelism across ranks (Split-KV: Efficient Context Parallelism for Training
Diffusion Drafters, Abstract and its table of context-parallel methods).

* The host LPT of chunks onto ranks (``splitkv_cp_plan``) equals the oracle's LPT over the chunk
  costs, on random costs and Graham's worst case.
* gloo, world size 2, on CPU: every rank reaches the same plan from the same anchors without any
  message, and the product's all-gather of the ranks' query-sized results (``gather_rank_results``),
  fed with each rank's oracle partial over its own chunks, merges to the single-pass oracle result.
* One GPU (``-m gpu``): the ranks' steps run one after another through the C ABI (cost of the rank,
  plan, forward, the rank's merge), then the merge over ranks; O and LSE match the oracle, for 1 to 4
  ranks, and each rank reads K/V only from its own chunks (the other rows hold a large value). The
  backward: each rank's share (``splitkv_attn_bwd_rank``) from the merged O and LSE, summed over the
  ranks, matches the oracle's gradients (1 to 3 ranks, bf16 and fp32).
* gloo, world size 2, on CPU: the gradient all-reduce (``reduce_rank_grads``) sums the ranks' parts.
* The rank backward's argument checks, on CPU.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import workloads as W
from oracle import attention as OA
from oracle import schedule as OS
from tests._util import anchors_per_sample, oracle_problem

B = pytest.importorskip("split_kv_lse_splitkv_b200.binding", reason="libsplitkv.so not built")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("n_ranks", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("seed", range(4))
def test_cp_plan_equals_oracle_lpt(n_ranks, seed):
    rng = np.random.default_rng(seed)
    costs = rng.integers(0, 200, size=int(rng.integers(1, 80)))
    costs[: min(5, len(costs))] = 7  # ties: lower chunk index first, lower rank first
    rank, load = B.splitkv_cp_plan(costs, n_ranks)
    iw, _, _, ol = OS.lpt(costs.tolist(), n_ranks)
    assert rank.tolist() == iw.tolist()
    assert load.tolist() == ol.tolist()


def test_cp_plan_graham_worst_case_and_errors():
    rank, load = B.splitkv_cp_plan([3, 3, 2, 2, 2], 2)
    assert sorted(load.tolist()) == [5, 7]  # LPT makespan 7 (the optimum is 6)
    with pytest.raises(B.SplitKVError):
        B.splitkv_cp_plan([1, -1], 2)
    with pytest.raises(B.SplitKVError):
        B.splitkv_cp_plan([1, 2], 0)


def _chunk_costs(inp):
    w = inp.workload
    _, _, chunk_costs = OS.costs_closed_form(anchors_per_sample(inp), w.seq_lens, w.chunk, w.key_tile,
                                             w.n_kv_heads, pack=w.blocks_per_item)
    return chunk_costs


def _oracle_rank_result(inp, chunk_rank, rank, n_ranks):
    """The rank's (O_r, LSE_r) by the oracle: merge of its chunks' partials (+ its blocks' own keys)."""
    w = inp.workload
    p = oracle_problem(inp)
    parts = OA.chunk_partials(p, w.chunk)
    nc = [-(-int(S) // w.chunk) for S in w.seq_lens]
    base = np.concatenate([[0], np.cumsum(nc)])
    mine = {}
    for (s, c, j, h), val in parts.items():
        owner = j % n_ranks if c < 0 else int(chunk_rank[base[s] + c])
        if owner == rank:
            mine[(s, c, j, h)] = val
    Nq, Hq, d = inp.q.shape
    O = np.zeros((Nq, Hq, d))
    L = np.full((Nq, Hq), -np.inf)
    groups = {}
    for (s, c, j, h), val in mine.items():
        groups.setdefault((j, h), []).append(val)
    for (j, h), vals in groups.items():
        r = p.rows(j)
        O[r, h], L[r, h] = OA.lse_merge([x[0] for x in vals], [x[1] for x in vals])
    return O, L


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir, n):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(n), RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from split_kv_lse_splitkv_b200 import cp
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    inp = W.make_inputs(W.scaled(W.get("drafter_s32k"), "cp_gloo", [2500, 1300], [3, 2], chunk=256, seed=31,
                                 n_q_heads=4, n_kv_heads=2, head_dim=16))
    chunk_rank, load = cp.cp_plan_chunks(_chunk_costs(inp), n)
    # The same plan on every rank, reached without any message.
    every = [torch.zeros_like(chunk_rank) for _ in range(n)]
    dist.all_gather(every, chunk_rank)
    assert all(torch.equal(every[0], x) for x in every)
    O_r, L_r = _oracle_rank_result(inp, chunk_rank.numpy(), rank, n)
    o_all, lse_all = cp.gather_rank_results(torch.from_numpy(O_r), torch.from_numpy(L_r))
    assert o_all.shape[0] == n and torch.equal(o_all[rank], torch.from_numpy(O_r))
    O, L = OA.lse_merge([o_all[r].numpy().reshape(-1, o_all.shape[-1]) for r in range(n)],
                        [lse_all[r].numpy().reshape(-1) for r in range(n)])
    O_ref, L_ref = OA.forward(oracle_problem(inp))
    err = max(float(np.abs(O.reshape(O_ref.shape) - O_ref).max()), float(np.abs(L.reshape(L_ref.shape) - L_ref).max()))
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(f"{err!r} {load.tolist()}")
    dist.barrier()
    dist.destroy_process_group()


def _reduce_main(rank, port, out_dir, n):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(n), RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from split_kv_lse_splitkv_b200 import cp
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    g = torch.Generator().manual_seed(rank)
    parts = [torch.randn(5, 4, 8, generator=g), torch.randn(5, 2, 8, generator=g), torch.randn(5, 2, 8, generator=g)]
    mine = [x.clone() for x in parts]
    cp.reduce_rank_grads(*mine)
    torch.save({"parts": parts, "reduced": mine}, os.path.join(out_dir, f"grads{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("n", [2, 3])
def test_gloo_ranks_gradient_reduce(tmp_path, n):
    mp.start_processes(_reduce_main, args=(_free_port(), str(tmp_path), n), nprocs=n, join=True, start_method="spawn")
    got = [torch.load(tmp_path / f"grads{r}.pt") for r in range(n)]
    for i in range(3):
        want = sum(got[r]["parts"][i] for r in range(n))
        for r in range(n):  # float32 sums of three terms: the library may add them in another order
            assert torch.allclose(got[r]["reduced"][i], want, rtol=0, atol=1e-6)


def test_rank_backward_argument_checks():
    p = B.make_problem([1024], [0, 4], 1, 1, 64, 16, 128, 128, 0.125, torch.float32)
    fake = torch.zeros(64, dtype=torch.uint8)
    ws = torch.empty(B.splitkv_workspace_size(p, 4), dtype=torch.uint8)
    for rank, n in ((-1, 2), (2, 2), (0, 0)):
        with pytest.raises(B.SplitKVError) as e:
            B.splitkv_attn_bwd_rank(p, *([fake] * 9), fake, rank, n, *([fake] * 6), ws, stream=0)
        assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:  # no chunk placement
        B.splitkv_attn_bwd_rank(p, *([fake] * 9), None, 0, 2, *([fake] * 6), ws, stream=0)
    assert e.value.code == B.EINVAL
    runs = B.make_problem([1024], [0, 4], 1, 1, 64, 16, 128, 128, 0.125, torch.float32, chunks_per_item=2)
    with pytest.raises(B.SplitKVError) as e:  # items must lie in one chunk
        B.splitkv_attn_bwd_rank(runs, *([fake] * 9), fake, 0, 2, *([fake] * 6), ws, stream=0)
    assert e.value.code == B.EUNSUPPORTED


@pytest.mark.parametrize("n", [2, 3])
def test_gloo_ranks_plan_gather_and_merge(tmp_path, n):
    mp.start_processes(_rank_main, args=(_free_port(), str(tmp_path), n), nprocs=n, join=True, start_method="spawn")
    for r in range(n):
        err, load = open(tmp_path / f"rank{r}.txt").read().split(" ", 1)
        assert float(err) < 1e-12, err


@pytest.mark.gpu
@pytest.mark.parametrize("n_ranks", [1, 2, 3, 4])
def test_ranks_on_one_gpu_match_the_oracle(n_ranks):
    from split_kv_lse_splitkv_b200.cp import ContextParallelSplitKV
    inp = W.make_inputs(W.scaled(W.get("drafter_s32k"), "cp_gpu", [5000, 3000], [5, 3], chunk=1024, seed=33))
    w = inp.workload
    counts = [int(inp.anchor_off[i + 1] - inp.anchor_off[i]) for i in range(len(w.seq_lens))]
    dev = {k: getattr(inp, k).cuda() for k in ("q", "k", "v", "kb", "vb")}
    anchors = inp.anchors.cuda()
    o_ranks, lse_ranks = [], []
    for r in range(n_ranks):
        cp = ContextParallelSplitKV(w.seq_lens, counts, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.chunk,
                                    w.key_tile, w.scale, w.torch_dtype, n_workers=8, rank=r, n_ranks=n_ranks)
        cp.plan(anchors)
        # This rank's K/V: only its own chunks' rows are real; the others hold a large value that would
        # spoil the result if any were read as a visible key (masked columns get P = 0 exactly).
        cr, parts, base = cp.chunk_rank.cpu(), [], 0
        for S in w.seq_lens:
            nc = -(-int(S) // w.chunk)
            parts.append(torch.repeat_interleave(cr[base:base + nc], w.chunk)[: int(S)])
            base += nc
        mine = (torch.cat(parts) == r).cuda()[:, None, None]
        k_r = torch.where(mine, dev["k"], torch.full_like(dev["k"], 256.0))
        v_r = torch.where(mine, dev["v"], torch.full_like(dev["v"], 256.0))
        o_r, lse_r = cp.local_forward(dev["q"], k_r, v_r, dev["kb"], dev["vb"], anchors)
        torch.cuda.synchronize()
        cp.skv.check_status()
        o_ranks.append(o_r)
        lse_ranks.append(lse_r)
        last = cp
    o, lse = last.combine(torch.stack(o_ranks), torch.stack(lse_ranks))
    torch.cuda.synchronize()
    last.skv.check_status()
    O, L = OA.forward(oracle_problem(inp))
    from tests._gpu import assert_close
    from tests._util import to_np
    assert_close("O (ranks)", to_np(o), O, w.dtype)
    assert_close("LSE (ranks)", to_np(lse), L, w.dtype)


@pytest.mark.gpu
@pytest.mark.parametrize("n_ranks,base", [(1, "drafter_s32k"), (2, "drafter_s32k"), (3, "drafter_s32k"), (2, "tiny_f32")])
def test_ranks_on_one_gpu_backward_matches_the_oracle(n_ranks, base):
    # Forward on one GPU, then each rank's share of the backward (its chunks' key tiles, its blocks' own
    # keys) with K/V rows of other ranks' chunks set to a large value; the sum of the shares is the
    # single-GPU backward.
    from split_kv_lse_splitkv_b200.cp import ContextParallelSplitKV
    kw = dict(chunk=1024, seed=35) if base == "drafter_s32k" else dict(chunk=128, seed=36)
    lens, cnts = ([5000, 3000], [5, 3]) if base == "drafter_s32k" else ([1024, 700], [4, 3])
    inp = W.make_inputs(W.scaled(W.get(base), "cp_bwd", lens, cnts, backward=True, **kw))
    w = inp.workload
    counts = [int(inp.anchor_off[i + 1] - inp.anchor_off[i]) for i in range(len(w.seq_lens))]
    dev = {k: getattr(inp, k).cuda() for k in ("q", "k", "v", "kb", "vb", "do")}
    anchors = inp.anchors.cuda()
    skv = B.SplitKV(w.seq_lens, counts, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.chunk, w.key_tile, w.scale,
                    w.torch_dtype, n_workers=8)
    o, lse = skv.forward(dev["q"], dev["k"], dev["v"], dev["kb"], dev["vb"], anchors)
    total = None
    for r in range(n_ranks):
        cp = ContextParallelSplitKV(w.seq_lens, counts, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.chunk,
                                    w.key_tile, w.scale, w.torch_dtype, n_workers=8, rank=r, n_ranks=n_ranks)
        cp.plan(anchors)
        cr, parts, base_c = cp.chunk_rank.cpu(), [], 0
        for S in w.seq_lens:
            nc = -(-int(S) // w.chunk)
            parts.append(torch.repeat_interleave(cr[base_c:base_c + nc], w.chunk)[: int(S)])
            base_c += nc
        mine = (torch.cat(parts) == r).cuda()[:, None, None]
        k_r = torch.where(mine, dev["k"], torch.full_like(dev["k"], 256.0))
        v_r = torch.where(mine, dev["v"], torch.full_like(dev["v"], 256.0))
        grads = cp.local_backward(dev["q"], k_r, v_r, dev["kb"], dev["vb"], o, lse, dev["do"], anchors)
        torch.cuda.synchronize()
        cp.skv.check_status()
        other = ~mine[:, 0, 0]  # key rows of other ranks' chunks: their dK, dV stay zero here
        if bool(other.any()):
            assert float(grads[1][other].abs().max()) == 0.0 and float(grads[2][other].abs().max()) == 0.0
        total = [g.clone() for g in grads] if total is None else [t + g for t, g in zip(total, grads)]
    from tests._gpu import assert_close
    from tests._util import to_np
    ref = OA.backward(oracle_problem(inp), to_np(inp.do))
    for name, g, rf in zip(("dQ", "dK", "dV", "dKb", "dVb"), total, ref):
        assert_close(name + " (ranks)", to_np(g), rf, w.dtype)
