"""LTE (contextualized Learnable Token Eviction) on B200: a C-ABI CUDA library
(liblte.so, sm_100a) and its Python binding.

``lte``   - one function per C entry point (argument marshalling only).
``layer`` - buffer allocation and the call sequence of one layer.
The binding loads liblte.so on import and fails if it is missing.
"""
from .lte import (LteError, lte_cache_init_from_prefill, lte_clear_device_error,  # noqa: F401
                  lte_decode_step, lte_evict_compact, lte_gla_decode_step, lte_gla_prefill,
                  lte_read_device_error, lte_score, lte_sparse_attn_prefill, lte_workspace_bytes,
                  version)
