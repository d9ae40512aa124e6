"""CPU oracle (test infrastructure only; never imported by the GPU library).

``lte_oracle``: retention CNN, eviction mask, compaction, attended sets,
sparse attention (prefill) and a slot-by-slot simulation of the decode cache.
``gla_oracle``: the gated linear-attention recurrence of the hybrid.
"""
