"""Split-KV hot path on one B200: Python binding of the C ABI in ``include/splitkv.h``.

The binding only marshals arguments (device pointers from torch tensors, the
problem description, the current CUDA stream) into ``libsplitkv.so``; every step
of the path runs in that library's kernels. The library is loaded on first use of
any name below; if it is not built, that raises ImportError: there is no fallback.
(``python -m split_kv_lse_splitkv_b200.build`` builds it without loading it.)

Entry points (same names as the C ABI): :func:`splitkv_query`,
:func:`splitkv_workspace_size`, :func:`splitkv_cost`, :func:`splitkv_plan_lpt`,
:func:`splitkv_attn_fwd`, :func:`splitkv_lse_merge`, :func:`splitkv_attn_bwd`,
:func:`splitkv_strerror`, :func:`splitkv_last_error`. :class:`SplitKV` strings them
together with torch-allocated buffers.
"""
_EXPORTS = (
    "DEV_ANCHOR_ORDER", "DEV_ANCHOR_RANGE", "DEV_BAD_COST", "DEV_BAD_PLAN", "DEV_SMEM_ALIGN", "DEV_TIMEOUT", "FWD_DEFAULT", "FWD_SIMT",
    "FWD_TEST_STARVE",
    "LIB_PATH", "SplitKV", "SplitKVError", "make_problem", "splitkv_attn_bwd", "splitkv_attn_fwd", "splitkv_cost",
    "splitkv_last_error", "splitkv_lse_merge", "splitkv_max_workers", "splitkv_cp_plan", "splitkv_cost_rank",
    "splitkv_lse_merge_rank", "splitkv_lse_merge_ranks", "splitkv_attn_bwd_rank", "ContextParallelSplitKV", "splitkv_plan_lpt", "splitkv_plan_lpt_noalloc", "splitkv_query", "splitkv_strerror",
    "splitkv_workspace_size",
)
__all__ = list(_EXPORTS)


def __getattr__(name):
    if name == "ContextParallelSplitKV":
        from . import cp
        return cp.ContextParallelSplitKV
    if name in _EXPORTS:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
