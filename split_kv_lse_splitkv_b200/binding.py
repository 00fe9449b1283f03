"""ctypes binding of libsplitkv.so: argument marshalling only (no arithmetic of the method here)."""
from __future__ import annotations

import ctypes
import math
import os
import warnings
from typing import Optional, Sequence

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsplitkv.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m split_kv_lse_splitkv_b200.build` (needs nvcc)")
_lib = ctypes.CDLL(LIB_PATH)

# Constants mirrored from include/splitkv.h.
OK, EINVAL, EUNSUPPORTED, ECUDA, ENOSPACE = 0, -1, -2, -3, -4
DEV_ANCHOR_ORDER, DEV_ANCHOR_RANGE, DEV_BAD_COST, DEV_BAD_PLAN, DEV_TIMEOUT = 0x1, 0x2, 0x4, 0x8, 0x10
DEV_SMEM_ALIGN = 0x20
F32, BF16 = 0, 1
FWD_DEFAULT, FWD_SIMT, FWD_TEST_STARVE = 0, 1, 0x100
MAX_BATCH = 64

_i32, _i64, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class Problem(ctypes.Structure):
    _fields_ = [
        ("batch", _i32),
        ("seq_len", ctypes.POINTER(_i64)),
        ("anchor_off", ctypes.POINTER(_i32)),
        ("n_q_heads", _i32),
        ("n_kv_heads", _i32),
        ("head_dim", _i32),
        ("block", _i32),
        ("chunk", _i32),
        ("key_tile", _i32),
        ("scale", _f32),
        ("dtype", _i32),
        ("blocks_per_item", _i32),
        ("chunks_per_item", _i32),
        ("item_overhead", _i32),
    ]


class Sizes(ctypes.Structure):
    _fields_ = [
        ("n_items_max", _i64),
        ("n_chunks", _i64),
        ("n_queries", _i64),
        ("total_keys", _i64),
        ("n_blocks", _i64),
        ("o_part_elems", _i64),
        ("lse_part_elems", _i64),
        ("max_cost", _i32),
        ("rows_per_item", _i32),
        ("ctas_per_worker", _i32),
    ]


_PP = ctypes.POINTER(Problem)
_SIGS = {
    "splitkv_query": (_i32, [_PP, ctypes.POINTER(Sizes)]),
    "splitkv_workspace_size": (_sz, [_PP, _i32]),
    "splitkv_max_workers": (_i32, [_PP, ctypes.POINTER(_i32)]),
    "splitkv_strerror": (ctypes.c_char_p, [_i32]),
    "splitkv_last_error": (ctypes.c_char_p, []),
    "splitkv_build_id": (ctypes.c_char_p, []),
    "splitkv_cost": (_i32, [_PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "splitkv_plan_lpt": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "splitkv_plan_lpt_noalloc": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp]),
    "splitkv_attn_fwd": (_i32, [_PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _vp,
                                _sz, _vp]),
    "splitkv_lse_merge": (_i32, [_PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "splitkv_attn_bwd": (_i32, [_PP] + [_vp] * 9 + [_vp] * 6 + [_vp, _sz, _vp]),
    "splitkv_attn_bwd_rank": (_i32, [_PP] + [_vp] * 10 + [_i32, _i32] + [_vp] * 6 + [_vp, _sz, _vp]),
    "splitkv_cp_plan": (_i32, [_vp, _i64, _i32, _vp, _vp]),
    "splitkv_cost_rank": (_i32, [_PP, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "splitkv_lse_merge_rank": (_i32, [_PP, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "splitkv_lse_merge_ranks": (_i32, [_PP, _i32, _vp, _vp, _vp, _vp, _vp, _vp]),
}
EXPORTS = tuple(_SIGS)
for _name, (_res, _args) in _SIGS.items():
    try:
        _fn = getattr(_lib, _name)
    except AttributeError:
        raise ImportError(f"{LIB_PATH} does not export {_name}: it was built from older sources; rebuild with "
                          "`python -m split_kv_lse_splitkv_b200.build`") from None
    _fn.restype = _res
    _fn.argtypes = _args


def library_build_id() -> str:
    """sha256 of the sources the loaded library was compiled from ("unknown" if its build supplied none)."""
    return _lib.splitkv_build_id().decode()


def _warn_if_stale() -> None:
    # A library built from other sources than those beside it runs other code than they say.
    try:
        from .build import source_digest
        want = source_digest()
    except (ImportError, OSError):  # no sources beside the library
        return
    got = library_build_id()
    if got != want:
        warnings.warn(f"{LIB_PATH} was built from other sources than those beside it (build id {got[:12]}, "
                      f"sources {want[:12]}): rebuild with `python -m split_kv_lse_splitkv_b200.build`",
                      RuntimeWarning, stacklevel=2)


_warn_if_stale()


class SplitKVError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = splitkv_last_error() if code in (ECUDA, ENOSPACE) else ""
        super().__init__(f"{where}: {splitkv_strerror(code)} ({code})" + (f" [{detail}]" if detail else ""))


def splitkv_last_error() -> str:
    return _lib.splitkv_last_error().decode()


def splitkv_strerror(code: int) -> str:
    return _lib.splitkv_strerror(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != OK:
        raise SplitKVError(code, where)


class ProblemHolder:
    """A ``splitkv_problem`` plus the host arrays it points to (kept alive with it)."""

    def __init__(self, seq_lens: Sequence[int], anchor_off: Sequence[int], n_q_heads: int, n_kv_heads: int,
                 head_dim: int, block: int, chunk: int, key_tile: int, scale: float, dtype: int,
                 blocks_per_item: int = 1, chunks_per_item: int = 1, item_overhead: int = 0):
        self.seq_arr = (_i64 * len(seq_lens))(*[int(x) for x in seq_lens])
        self.off_arr = (_i32 * len(anchor_off))(*[int(x) for x in anchor_off])
        self.struct = Problem(len(seq_lens), self.seq_arr, self.off_arr, n_q_heads, n_kv_heads, head_dim, block,
                              chunk, key_tile, float(scale), dtype, int(blocks_per_item), int(chunks_per_item),
                              int(item_overhead))

    @property
    def ptr(self):
        return ctypes.byref(self.struct)


def make_problem(seq_lens, anchor_off, n_q_heads, n_kv_heads, head_dim, block=16, chunk=1024, key_tile=128,
                 scale=None, dtype=torch.bfloat16, blocks_per_item=1, chunks_per_item=1,
                 item_overhead=0) -> ProblemHolder:
    code = F32 if dtype == torch.float32 else BF16 if dtype == torch.bfloat16 else None
    if code is None:
        raise SplitKVError(EUNSUPPORTED, f"dtype {dtype}")
    scale = 1.0 / math.sqrt(head_dim) if scale is None else scale
    return ProblemHolder(seq_lens, anchor_off, n_q_heads, n_kv_heads, head_dim, block, chunk, key_tile, scale, code,
                         blocks_per_item, chunks_per_item, item_overhead)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(getattr(stream, "cuda_stream", stream)))


# ------------------------------------------------------------------ C ABI, one to one
def splitkv_query(problem: ProblemHolder) -> Sizes:
    out = Sizes()
    _check(_lib.splitkv_query(problem.ptr, ctypes.byref(out)), "splitkv_query")
    return out


def splitkv_max_workers(problem: ProblemHolder) -> int:
    """Workers whose queues all run at once on the current device (SMs, or co-resident SM pairs)."""
    out = _i32(0)
    _check(_lib.splitkv_max_workers(problem.ptr, ctypes.byref(out)), "splitkv_max_workers")
    return int(out.value)


def splitkv_workspace_size(problem: ProblemHolder, n_workers: int) -> int:
    return int(_lib.splitkv_workspace_size(problem.ptr, int(n_workers)))


def splitkv_cost(problem, anchors, item_id, item_cost, chunk_cost, n_items, status, workspace, stream=None):
    _check(_lib.splitkv_cost(problem.ptr, _p(anchors), _p(item_id), _p(item_cost), _p(chunk_cost), _p(n_items),
                             _p(status), _p(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream)), "splitkv_cost")


def splitkv_plan_lpt(item_cost, n_items, max_items, max_cost, n_workers, item_worker, queue_off, queue_items, load,
                     status, workspace, stream=None):
    _check(_lib.splitkv_plan_lpt(_p(item_cost), _p(n_items), int(max_items), int(max_cost), int(n_workers),
                                 _p(item_worker), _p(queue_off), _p(queue_items), _p(load), _p(status),
                                 _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "splitkv_plan_lpt")


def splitkv_plan_lpt_noalloc(item_cost, n_items, max_items, max_cost, n_workers, item_worker, queue_off, queue_items,
                             load, status, stream=None):
    """splitkv_plan_lpt without a workspace: scratch comes from a static array inside the library
    (for callers that cannot allocate device memory, e.g. during CUDA graph capture)."""
    _check(_lib.splitkv_plan_lpt_noalloc(_p(item_cost), _p(n_items), int(max_items), int(max_cost), int(n_workers),
                                         _p(item_worker), _p(queue_off), _p(queue_items), _p(load), _p(status),
                                         _stream(stream)), "splitkv_plan_lpt_noalloc")


def splitkv_attn_fwd(problem, q, k, v, kb, vb, anchors, item_id, queue_off, queue_items, n_workers, o_part,
                     lse_part, status, flags=FWD_DEFAULT, workspace=None, stream=None):
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.splitkv_attn_fwd(problem.ptr, _p(q), _p(k), _p(v), _p(kb), _p(vb), _p(anchors), _p(item_id),
                                 _p(queue_off), _p(queue_items), int(n_workers), _p(o_part), _p(lse_part), _p(status),
                                 int(flags), _p(workspace), nbytes, _stream(stream)), "splitkv_attn_fwd")


def splitkv_lse_merge(problem, o_part, lse_part, anchors, o, lse, status, stream=None):
    _check(_lib.splitkv_lse_merge(problem.ptr, _p(o_part), _p(lse_part), _p(anchors), _p(o), _p(lse), _p(status),
                                  _stream(stream)), "splitkv_lse_merge")


def splitkv_attn_bwd(problem, q, k, v, kb, vb, o, lse, dout, anchors, dq, dk, dv, dkb, dvb, status, workspace,
                     stream=None):
    _check(_lib.splitkv_attn_bwd(problem.ptr, _p(q), _p(k), _p(v), _p(kb), _p(vb), _p(o), _p(lse), _p(dout),
                                 _p(anchors), _p(dq), _p(dk), _p(dv), _p(dkb), _p(dvb), _p(status), _p(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)), "splitkv_attn_bwd")


def splitkv_attn_bwd_rank(problem, q, k, v, kb, vb, o, lse, dout, anchors, chunk_rank, rank, n_ranks, dq, dk, dv, dkb,
                          dvb, status, workspace, stream=None):
    _check(_lib.splitkv_attn_bwd_rank(problem.ptr, _p(q), _p(k), _p(v), _p(kb), _p(vb), _p(o), _p(lse), _p(dout),
                                      _p(anchors), _p(chunk_rank), int(rank), int(n_ranks), _p(dq), _p(dk), _p(dv),
                                      _p(dkb), _p(dvb), _p(status), _p(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)),
           "splitkv_attn_bwd_rank")


def splitkv_cp_plan(chunk_cost, n_ranks):
    """Host LPT of chunks onto ranks: (chunk_rank int32[n_chunks], rank_load int64[n_ranks]) as CPU tensors."""
    cost = torch.as_tensor(chunk_cost, dtype=torch.int64).cpu().contiguous()
    rank = torch.empty(cost.numel(), dtype=torch.int32)
    load = torch.empty(int(n_ranks), dtype=torch.int64)
    _check(_lib.splitkv_cp_plan(_p(cost), int(cost.numel()), int(n_ranks), _p(rank), _p(load)), "splitkv_cp_plan")
    return rank, load


def splitkv_cost_rank(problem, anchors, chunk_rank, rank, n_ranks, item_id, item_cost, chunk_cost, n_items, status,
                      workspace, stream=None):
    _check(_lib.splitkv_cost_rank(problem.ptr, _p(anchors), _p(chunk_rank), int(rank), int(n_ranks), _p(item_id),
                                  _p(item_cost), _p(chunk_cost), _p(n_items), _p(status), _p(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)), "splitkv_cost_rank")


def splitkv_lse_merge_rank(problem, o_part, lse_part, anchors, chunk_rank, rank, n_ranks, o_r, lse_r, status,
                           stream=None):
    _check(_lib.splitkv_lse_merge_rank(problem.ptr, _p(o_part), _p(lse_part), _p(anchors), _p(chunk_rank), int(rank),
                                       int(n_ranks), _p(o_r), _p(lse_r), _p(status), _stream(stream)),
           "splitkv_lse_merge_rank")


def splitkv_lse_merge_ranks(problem, n_ranks, o_ranks, lse_ranks, o, lse, status, stream=None):
    _check(_lib.splitkv_lse_merge_ranks(problem.ptr, int(n_ranks), _p(o_ranks), _p(lse_ranks), _p(o), _p(lse),
                                        _p(status), _stream(stream)), "splitkv_lse_merge_ranks")


# ------------------------------------------------------------------ convenience: the whole path
class SplitKV:
    """Buffers and calls for one problem shape: cost -> LPT plan -> partial forward -> merge (-> backward).

    All device buffers are allocated once here with torch; the calls enqueue work on the
    current stream and never synchronize. ``anchor_counts`` fixes the number of blocks per sample;
    the anchor values themselves are device data passed to :meth:`plan`.
    """

    def __init__(self, seq_lens, anchor_counts, n_q_heads, n_kv_heads, head_dim, block=16, chunk=1024,
                 key_tile=128, scale=None, dtype=torch.bfloat16, n_workers=None, device="cuda", blocks_per_item=1,
                 chunks_per_item=1, item_overhead=0):
        off = [0]
        for c in anchor_counts:
            off.append(off[-1] + int(c))
        self.device = torch.device(device)
        self.dtype = dtype
        self.n_q_heads, self.n_kv_heads, self.head_dim = int(n_q_heads), int(n_kv_heads), int(head_dim)
        self.problem = make_problem(seq_lens, off, n_q_heads, n_kv_heads, head_dim, block, chunk, key_tile, scale,
                                    dtype, blocks_per_item, chunks_per_item, item_overhead)
        self.blocks_per_item = int(blocks_per_item) or 1
        self.chunks_per_item = int(chunks_per_item) or 1
        self.sizes = splitkv_query(self.problem)
        if n_workers is None:  # one queue per SM, or per co-resident pair of SMs for 256-row items
            with torch.cuda.device(self.device):
                n_workers = splitkv_max_workers(self.problem)
        self.n_workers = int(n_workers)
        s = self.sizes
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        nmax = max(1, int(s.n_items_max))
        self.status = torch.zeros(1, **i32)
        self.item_id = torch.empty(nmax, **i32)
        self.item_cost = torch.empty(nmax, **i32)
        self.chunk_cost = torch.empty(max(1, int(s.n_chunks)), dtype=torch.int64, device=dev)
        self.n_items = torch.zeros(1, **i32)
        self.item_worker = torch.empty(nmax, **i32)
        self.queue_off = torch.empty(self.n_workers + 1, **i32)
        self.queue_items = torch.empty(nmax, **i32)
        self.load = torch.empty(self.n_workers, dtype=torch.int64, device=dev)
        ws = splitkv_workspace_size(self.problem, self.n_workers)
        if ws == 0:
            raise SplitKVError(EINVAL, "splitkv_workspace_size")
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.o_part = torch.empty(max(8, int(s.o_part_elems)), dtype=dtype, device=dev)  # problem dtype
        self.lse_part = torch.empty(max(1, int(s.lse_part_elems)), dtype=torch.float32, device=dev)

    # -- steps
    def cost(self, anchors, stream=None):
        splitkv_cost(self.problem, anchors, self.item_id, self.item_cost, self.chunk_cost, self.n_items, self.status,
                     self.workspace, stream)

    def plan_lpt(self, stream=None):
        splitkv_plan_lpt(self.item_cost, self.n_items, int(self.sizes.n_items_max), int(self.sizes.max_cost),
                         self.n_workers, self.item_worker, self.queue_off, self.queue_items, self.load, self.status,
                         self.workspace, stream)

    def plan(self, anchors, stream=None):
        self.cost(anchors, stream)
        self.plan_lpt(stream)

    def attn_fwd(self, q, k, v, kb, vb, anchors, flags=FWD_DEFAULT, stream=None):
        splitkv_attn_fwd(self.problem, q, k, v, kb, vb, anchors, self.item_id, self.queue_off, self.queue_items,
                         self.n_workers, self.o_part, self.lse_part, self.status, flags, self.workspace, stream)

    def lse_merge(self, anchors, o=None, lse=None, stream=None):
        Nq, Hq, d = int(self.sizes.n_queries), self.n_q_heads, self.head_dim
        if o is None:
            o = torch.empty(Nq, Hq, d, dtype=self.dtype, device=self.device)
        if lse is None:
            lse = torch.empty(Nq, Hq, dtype=torch.float32, device=self.device)
        splitkv_lse_merge(self.problem, self.o_part, self.lse_part, anchors, o, lse, self.status, stream)
        return o, lse

    def forward(self, q, k, v, kb, vb, anchors, flags=FWD_DEFAULT, plan=True, o=None, lse=None, stream=None):
        if plan:
            self.plan(anchors, stream)
        self.attn_fwd(q, k, v, kb, vb, anchors, flags, stream)
        return self.lse_merge(anchors, o, lse, stream)

    def backward(self, q, k, v, kb, vb, o, lse, dout, anchors, grads=None, stream=None):
        """dQ, dK, dV, dKb, dVb (float32), from the forward's o and lse (no plan needed)."""
        if grads is None:
            f = dict(dtype=torch.float32, device=self.device)
            grads = (torch.empty(q.shape, **f), torch.empty(k.shape, **f), torch.empty(v.shape, **f),
                     torch.empty(kb.shape, **f), torch.empty(vb.shape, **f))
        dq, dk, dv, dkb, dvb = grads
        splitkv_attn_bwd(self.problem, q, k, v, kb, vb, o, lse, dout, anchors, dq, dk, dv, dkb, dvb, self.status,
                         self.workspace, stream)
        return grads

    # -- host-side reads (synchronizing; for tests and reports)
    def status_value(self) -> int:
        return int(self.status.item())

    def check_status(self):
        st = self.status_value()
        if st:
            raise RuntimeError(f"device status word 0x{st:x}")

    def o_part_view(self):
        """Partials as [slots, d/E, rows, E] (problem dtype, E = 16 bytes / element size) and their LSEs
        as [slots, rows]: chunk items first (n_items_max slots), then the self partials, slot
        n_items_max + j*Hkv + g."""
        R, d = int(self.sizes.rows_per_item), self.head_dim
        E = 16 // self.o_part.element_size()
        n = int(self.sizes.lse_part_elems) // R
        return self.o_part[: n * R * d].view(n, d // E, R, E), self.lse_part[: n * R].view(n, R)
