"""CPU oracle of the paged KV-cache path (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package. The product package never does; the two share no code.
"""
from .block_hash import block_hashes
from .paged_attention import (bf16_bits_to_f64, compare, copy_blocks, decode, gather_sequence,
                              physical_row, prefill, softmax_attention, store_kvcache)

__all__ = ["bf16_bits_to_f64", "compare", "decode", "gather_sequence", "physical_row", "prefill",
           "softmax_attention", "store_kvcache", "copy_blocks", "block_hashes"]
