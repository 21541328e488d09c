"""QUOKA query-oriented KV selection + sparse GQA attention for NVIDIA B200.

The compute path is libquoka.so (hand-written sm_100a CUDA kernels behind a
C ABI, declared in include/quoka.h); this package holds that library's
sources, its build script, a thin ctypes binding with the same entry-point
names, and the seeded synthetic input generators.

The binding is imported lazily so that the input generators can be used
without the built library.
"""

__all__ = [
    "quoka_workspace_size",
    "quoka_select_workspace_size",
    "quoka_attn_workspace_size",
    "quoka_decode_workspace_size",
    "quoka_decode_attn",
    "quoka_select",
    "quoka_gather_kv",
    "quoka_sparse_gqa_attn",
    "quoka_sparse_gqa_attn_gathered",
    "quoka_prefill_chunk",
    "quoka_get_device_status",
    "quoka_get_device_fault_site",
    "quoka_debug_set_wait_hooks",
    "quoka_status_string",
    "QuokaError",
    "quoka_select_static",
    "quoka_shard_candidate_scores",
    "quoka_shard_interleave",
    "quoka_topk",
    "quoka_shard_take",
    "quoka_combine_partials",
]


def __getattr__(name):
    if name in __all__ or name in ("load", "workspace_for", "tensor_view"):
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
