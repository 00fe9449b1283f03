"""The C ABI on a machine without a GPU: the library loads, exports every entry point that
include/splitkv.h declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "splitkv.h")

skv = pytest.importorskip("split_kv_lse_splitkv_b200", reason="libsplitkv.so not built")
from split_kv_lse_splitkv_b200 import binding as B  # noqa: E402


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(splitkv_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("splitkv_cost", "splitkv_plan_lpt", "splitkv_attn_fwd", "splitkv_lse_merge", "splitkv_attn_bwd"):
        assert n in names


def test_every_declared_symbol_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (splitkv_\w+)", out))
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(B._lib, n)
    assert set(B.EXPORTS) == set(declared_functions())
    # nothing else leaks out of the library's namespace
    assert all(n.startswith("splitkv_") for n in exported)


def prob(**kw):
    args = dict(seq_lens=[1024], anchor_off=[0, 4], n_q_heads=1, n_kv_heads=1, head_dim=64, block=16, chunk=128,
                key_tile=128, scale=0.125, dtype=torch.float32)
    args.update(kw)
    return B.make_problem(args.pop("seq_lens"), args.pop("anchor_off"), **args)


def test_query_sizes():
    s = B.splitkv_query(prob(seq_lens=[1000, 300], anchor_off=[0, 3, 5], n_q_heads=8, n_kv_heads=2, chunk=256))
    # items: sample 0: ceil(1000/256)=4 chunks * 2 heads * 3 blocks; sample 1: 2 chunks * 2 * 2
    assert s.n_items_max == 4 * 2 * 3 + 2 * 2 * 2
    assert s.n_chunks == 6 and s.n_queries == 80 and s.total_keys == 1300 and s.n_blocks == 5
    assert s.rows_per_item == 16 * 4 and s.max_cost == 2
    # partial slots: every item, then one self partial per (block, kv head)
    assert s.o_part_elems == (s.n_items_max + 5 * 2) * 64 * 64 and s.lse_part_elems == (s.n_items_max + 5 * 2) * 64
    assert B.splitkv_workspace_size(prob(), 4) > 0
    # two blocks per query tile: sample 0 has 3 blocks (2 tiles), sample 1 has 2 (1 tile)
    s2 = B.splitkv_query(prob(seq_lens=[1000, 300], anchor_off=[0, 3, 5], n_q_heads=8, n_kv_heads=2, chunk=256,
                              blocks_per_item=2))
    assert s2.n_items_max == 4 * 2 * 2 + 2 * 2 * 1 and s2.rows_per_item == 2 * 16 * 4
    assert s2.o_part_elems == (s2.n_items_max + 5 * 2) * 128 * 64


def test_query_sizes_with_runs_of_chunks():
    # Items over runs of 3 chunks: sample 0 has ceil(4/3) = 2 runs, sample 1 ceil(2/3) = 1; the chunk costs
    # (n_chunks) stay per chunk, the largest item cost is 3 chunks' key tiles.
    s = B.splitkv_query(prob(seq_lens=[1000, 300], anchor_off=[0, 3, 5], n_q_heads=8, n_kv_heads=2, chunk=256,
                             chunks_per_item=3))
    assert s.n_items_max == 2 * 2 * 3 + 1 * 2 * 2
    assert s.n_chunks == 6 and s.max_cost == 6
    assert s.o_part_elems == (s.n_items_max + 5 * 2) * 64 * 64
    with pytest.raises(B.SplitKVError) as e:  # more than 64 key tiles per item
        B.splitkv_query(prob(chunk=128 * 32, chunks_per_item=3))
    assert e.value.code == B.EUNSUPPORTED
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_query(prob(chunks_per_item=-1))
    assert e.value.code == B.EINVAL
    # A per-item constant of the cost raises the largest cost by itself.
    assert B.splitkv_query(prob(chunk=256, chunks_per_item=3, item_overhead=5)).max_cost == 6 + 5
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_query(prob(chunk=128 * 32, chunks_per_item=2, item_overhead=1))
    assert e.value.code == B.EUNSUPPORTED
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_query(prob(item_overhead=-1))
    assert e.value.code == B.EINVAL


def test_query_sizes_with_samples_without_anchors():
    # A sample without anchors has no block and no item; its keys still count (they sit between the
    # other samples' keys in K and V). A problem without any anchor is valid and empty.
    s = B.splitkv_query(prob(seq_lens=[1000, 700, 300], anchor_off=[0, 3, 3, 5], n_q_heads=8, n_kv_heads=2,
                             chunk=256))
    assert s.n_items_max == 4 * 2 * 3 + 0 + 2 * 2 * 2
    assert s.n_chunks == 4 + 3 + 2 and s.total_keys == 2000 and s.n_blocks == 5 and s.n_queries == 80
    e = B.splitkv_query(prob(seq_lens=[1000], anchor_off=[0, 0]))
    assert e.n_items_max == 0 and e.n_blocks == 0 and e.n_queries == 0 and e.o_part_elems == 0
    assert B.splitkv_workspace_size(prob(seq_lens=[1000], anchor_off=[0, 0]), 4) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(n_kv_heads=3, n_q_heads=4), B.EINVAL),          # Hkv does not divide Hq
    (dict(chunk=100), B.EUNSUPPORTED),                    # chunk not a multiple of key_tile
    (dict(chunk=128 * 65), B.EUNSUPPORTED),               # more than 64 key tiles per chunk
    (dict(head_dim=130), B.EUNSUPPORTED),
    (dict(head_dim=6), B.EUNSUPPORTED),
    (dict(scale=-1.0), B.EINVAL),
    (dict(seq_lens=[0]), B.EINVAL),
    (dict(anchor_off=[1, 4]), B.EINVAL),
    (dict(block=64), B.EUNSUPPORTED),
])
def test_bad_problems_are_rejected(kw, code):
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_query(prob(**kw))
    assert e.value.code == code
    assert B.splitkv_workspace_size(prob(**kw), 4) == 0


def test_bad_batch_and_workers():
    p = prob()
    p.struct.batch = 0
    with pytest.raises(B.SplitKVError):
        B.splitkv_query(p)
    assert B.splitkv_workspace_size(prob(), 0) == 0
    assert B.splitkv_workspace_size(prob(), 2000) == 0


def test_null_pointers_and_small_workspace_rejected_before_launch():
    p = prob()
    ws = torch.empty(B.splitkv_workspace_size(p, 4), dtype=torch.uint8)
    fake = torch.empty(64, dtype=torch.int32)  # host memory: never dereferenced, the calls fail first
    i64 = torch.empty(64, dtype=torch.int64)
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_cost(p, None, fake, fake, i64, fake, fake, ws, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_cost(p, fake, fake, fake, i64, fake, fake, ws[:1], stream=0)
    assert e.value.code == B.ENOSPACE
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_plan_lpt(fake, fake, 64, 0, 4, fake, fake, fake, i64, fake, ws, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_plan_lpt(fake, fake, 64, 1, 4096, fake, fake, fake, i64, fake, ws, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_attn_fwd(p, None, fake, fake, fake, fake, fake, fake, fake, fake, 4, fake, fake, fake, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:  # missing kb
        B.splitkv_attn_fwd(p, fake, fake, fake, None, fake, fake, fake, fake, fake, 4, fake, fake, fake, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:  # unknown flag
        B.splitkv_attn_fwd(p, fake, fake, fake, fake, fake, fake, fake, fake, fake, 4, fake, fake, fake, flags=8,
                           stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:  # misaligned q
        B.splitkv_attn_fwd(p, fake[1:], fake, fake, fake, fake, fake, fake, fake, fake, 4, fake, fake, fake, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:  # misaligned vb
        B.splitkv_attn_fwd(p, fake, fake, fake, fake, fake[1:], fake, fake, fake, fake, 4, fake, fake, fake, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:  # the tensor-core forward needs its workspace (pool counter)
        B.splitkv_attn_fwd(prob(head_dim=128, dtype=torch.bfloat16), *([fake] * 9), 4, fake, fake, fake, stream=0)
    assert e.value.code == B.ENOSPACE
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_lse_merge(p, fake, fake, fake, None, fake, fake, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:  # misaligned o
        B.splitkv_lse_merge(p, fake, fake, fake, fake[1:], fake, fake, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_attn_bwd(p, *([fake] * 9), *([fake] * 6), ws[:1], stream=0)
    assert e.value.code == B.ENOSPACE
    # bf16, d = 128: the tensor-core backward needs 16-byte aligned tensors.
    pb = prob(head_dim=128, dtype=torch.bfloat16)
    wsb = torch.empty(B.splitkv_workspace_size(pb, 4), dtype=torch.uint8)
    with pytest.raises(B.SplitKVError) as e:  # no dq
        B.splitkv_attn_bwd(pb, *([fake] * 9), None, *([fake] * 5), wsb, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:  # misaligned dk
        B.splitkv_attn_bwd(pb, *([fake] * 9), fake, fake[1:], *([fake] * 4), wsb, stream=0)
    assert e.value.code == B.EINVAL
    with pytest.raises(B.SplitKVError) as e:
        B.splitkv_attn_bwd(pb, *([fake] * 9), *([fake] * 6), wsb[:16], stream=0)
    assert e.value.code == B.ENOSPACE


def test_strerror():
    assert B.splitkv_strerror(0) == "ok"
    assert "workspace" in B.splitkv_strerror(B.ENOSPACE)
    assert B.splitkv_strerror(12345) == "unknown status"


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_problem_without_anchors_needs_no_query_buffers(dtype, d):
    # No anchor at all: nothing to compute. The forward (tensor-core or CUDA-core path) and the merge
    # accept empty (NULL) query-side buffers and return before any CUDA call, so this runs anywhere.
    p = prob(seq_lens=[1000], anchor_off=[0, 0], n_q_heads=8, n_kv_heads=2, head_dim=d, chunk=256, dtype=dtype)
    host = torch.empty(64, dtype=torch.int32)  # never dereferenced: the calls return before any access
    ws = torch.empty(B.splitkv_workspace_size(p, 4), dtype=torch.uint8)
    h = B._p(host)
    rc = B._lib.splitkv_attn_fwd(p.ptr, None, h, h, None, None, None, h, h, h, 4, h, h, h, B.FWD_DEFAULT, B._p(ws),
                                 ws.numel(), None)
    assert rc == B.OK, B.splitkv_strerror(rc)
    rc = B._lib.splitkv_lse_merge(p.ptr, h, h, None, None, None, h, None)
    assert rc == B.OK, B.splitkv_strerror(rc)
    # With anchors, the same NULL query buffers are refused.
    p1 = prob(seq_lens=[1000], anchor_off=[0, 2], n_q_heads=8, n_kv_heads=2, head_dim=d, chunk=256, dtype=dtype)
    rc = B._lib.splitkv_attn_fwd(p1.ptr, None, h, h, None, None, h, h, h, h, 4, h, h, h, B.FWD_DEFAULT, B._p(ws),
                                 ws.numel(), None)
    assert rc == B.EINVAL
    rc = B._lib.splitkv_lse_merge(p1.ptr, h, h, h, None, None, h, None)
    assert rc == B.EINVAL


def test_library_built_from_these_sources():
    # The build id compiled into libsplitkv.so is the digest of the sources beside it: a library left over
    # from other sources (edited, reverted or checked out after the build) fails here and warns on import.
    from split_kv_lse_splitkv_b200 import build
    assert B.library_build_id() == build.source_digest()
