"""splitkv_plan_lpt_noalloc: the planner entry point that allocates nothing.

Some callers cannot call cudaMalloc — code that runs while a CUDA graph is being captured, or inside a
framework whose caching allocator owns all device memory. For them the library offers a planner whose
scratch is a fixed array in the library's own device memory. These tests check, through the C ABI,
that it returns exactly the plan of the workspace-taking splitkv_plan_lpt on two calls in a row (the
array keeps the previous call's contents), and that it refuses a problem too large for the array.
This file is collected last on purpose: it runs after every other test, and also passes on its own.
"""
import re

import pytest
import torch

import workloads as W

B = pytest.importorskip("split_kv_lse_splitkv_b200.binding", reason="libsplitkv.so not built")


def test_noalloc_refuses_problems_beyond_its_static_scratch():
    fake = torch.empty(64, dtype=torch.int32)  # never touched: the call is refused on the host
    i64 = torch.empty(64, dtype=torch.int64)
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_plan_lpt_noalloc(fake, fake, 40_000_000, 64, 1024, fake, fake, fake, i64, fake, stream=0)
    assert e.value.code == B.ENOSPACE
    msg = str(e.value)
    assert "static array" in msg
    nums = [int(x) for x in re.findall(r"\d+", msg)]
    assert 4 << 20 in nums and any(x > 4 << 20 for x in nums), msg  # both sizes, the need above the array


def test_noalloc_accepts_the_largest_cost_on_every_sm():
    # max_cost 64 (chunk = 64 key tiles) on 148 queues with 200k items fits the static array: the call
    # passes the size check and, on a host without a GPU, fails only at the device lookup (ECUDA).
    # With a GPU these host tensors would reach a launch, so the case runs on GPU-less hosts only; the
    # GPU test below plans a max_cost 64 problem on 148 queues through this entry point.
    if torch.cuda.is_available():
        pytest.skip("host-only check of the size limit")
    fake = torch.empty(64, dtype=torch.int32)
    i64 = torch.empty(64, dtype=torch.int64)
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_plan_lpt_noalloc(fake, fake, 200_000, 64, 148, fake, fake, fake, i64, fake, stream=0)
    assert e.value.code == B.ECUDA, str(e.value)


def _plans(name, base, seq_lens, counts, chunk, runs=None):
    w = W.scaled(W.get(base), name, seq_lens, counts, chunk=chunk, seed=21,
                 **({} if runs is None else {"chunks_per_item": runs}))
    inp = W.make_inputs(w)
    cnt = [int(inp.anchor_off[i + 1] - inp.anchor_off[i]) for i in range(len(w.seq_lens))]
    skv = B.SplitKV(w.seq_lens, cnt, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.chunk, w.key_tile, w.scale,
                    w.torch_dtype, device="cuda", blocks_per_item=w.blocks_per_item,
                    chunks_per_item=w.chunks_per_item)
    skv.cost(inp.anchors.cuda())
    skv.plan_lpt()
    ref = [t.clone() for t in (skv.item_worker, skv.queue_off, skv.queue_items, skv.load)]
    outs = []
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        got = (torch.full_like(skv.item_worker, -7), torch.full_like(skv.queue_off, -7),
               torch.full_like(skv.queue_items, -7), torch.full_like(skv.load, -7))
        B.splitkv_plan_lpt_noalloc(skv.item_cost, skv.n_items, int(skv.sizes.n_items_max), int(skv.sizes.max_cost),
                                   skv.n_workers, *got, skv.status)
        outs.append(got)
    torch.cuda.synchronize()
    assert skv.status_value() == 0
    n = int(skv.n_items.item())
    return ref, outs, n


@pytest.mark.gpu
@pytest.mark.parametrize("case", [
    ("small", "drafter_s32k", [5000], [7], 1024),
    ("skewed", "skewed_s256k", [262144], [256], 2048),
    ("batch", "train_4x64k", [65536] * 4, [32, 64, 96, 128], 1024),
    ("wide_chunks", "drafter_s32k", [131072], [256], 8192, 1),  # max_cost 64 on 148 queues
])
def test_noalloc_plan_equals_workspace_plan(case):
    ref, outs, n = _plans(*case)
    for got in outs:
        assert torch.equal(got[0][:n], ref[0][:n])      # item_worker
        assert torch.equal(got[1], ref[1])              # queue_off
        assert torch.equal(got[2][:n], ref[2][:n])      # queue_items
        assert torch.equal(got[3], ref[3])              # load
