"""Float64 CPU oracle for GVA decode (TEST INFRASTRUCTURE).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import
this package.  The CUDA product path never does, and fails loudly without its
compiled library instead of falling back here.
"""
from .gva_oracle import (absorbed_query, append_cache, cache_scalars_gqa, cache_scalars_gva,
                         gqa_append_cache, gqa_decode, gva_decode, gva_decode_multi, rope, round_to_bf16, round_to_storage)

__all__ = ["absorbed_query", "append_cache", "cache_scalars_gqa", "cache_scalars_gva",
           "gqa_append_cache", "gqa_decode", "gva_decode", "gva_decode_multi", "rope", "round_to_bf16", "round_to_storage"]
