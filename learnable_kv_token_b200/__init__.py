"""LTE (contextualized Learnable Token Eviction) on B200: a C-ABI CUDA library
(liblte.so, sm_100a) and its Python binding.

``lte``   - one function per C entry point (argument marshalling only); importing
            it loads liblte.so and fails if the library is missing.
``layer`` - buffer allocation and the call sequence of one layer.
``build`` - compiles liblte.so (importable without the library).
"""
_LAZY = ("LteError", "lte_cache_init_from_prefill", "lte_clear_device_error", "lte_decode_step",
         "lte_decode_step_noalloc", "lte_evict_compact", "lte_gla_decode_step", "lte_gla_prefill",
         "lte_read_device_error", "lte_retained_lifetimes", "lte_score", "lte_score_backward",
         "lte_score_backward_workspace_bytes", "lte_sparse_attn_backward",
         "lte_sparse_attn_prefill", "lte_workspace_bytes",
         "version")


def __getattr__(name):
    if name in _LAZY:
        from . import lte
        return getattr(lte, name)
    raise AttributeError(name)
