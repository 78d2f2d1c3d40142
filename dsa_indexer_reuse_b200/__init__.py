"""B200 (sm_100a) DeepSeek-Sparse-Attention hot path with IndexCache
cross-layer index reuse.

This package is a thin Python binding over the C ABI of ``libindexcache.so``
(declared in ``include/indexcache.h``). Every step of the path runs in the
library's CUDA kernels; the binding only checks tensor metadata, allocates
outputs and workspace with PyTorch, and passes raw pointers and the current
CUDA stream. There is no CPU fallback: touching any entry point when the
library is missing raises ImportError.

Entry points (same names as the C ABI, without the ``ic_`` prefix):
    resolve_pattern, indexer_topk, sparse_attn, layer_stack,
    layer_stack_host (tensors in host memory, copies overlapped),
    indexer_workspace_size, sparse_attn_workspace_size,
    layer_stack_workspace_size, get_device_status, debug_expire_wait,
    topk_overlap, search_pattern, greedy_pattern (pattern tools), and
    overlap_matrix (layer x layer ratios), pattern_score (the search
    objective of one pattern), and
    distill_target (the multi-layer distillation target and KL of one Full layer)
    with distill_target_workspace_size.
The submodule ``workloads`` (seeded synthetic inputs) needs no library.
"""

_EXPORTS = (
    "BF16", "F32", "FP8_E4M3", "IcError", "LIB_PATH", "STATUS", "StackCall", "debug_expire_wait",
    "get_device_status", "indexer_topk", "indexer_workspace_size", "layer_stack",
    "layer_stack_workspace_size", "lib", "resolve_pattern", "sparse_attn",
    "sparse_attn_workspace_size", "version", "topk_overlap", "overlap_matrix", "search_pattern",
    "greedy_pattern", "pattern_score", "StackHostCall", "layer_stack_host", "distill_target",
    "distill_target_workspace_size",
)


def __getattr__(name):
    if name in _EXPORTS:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)


__all__ = list(_EXPORTS)
