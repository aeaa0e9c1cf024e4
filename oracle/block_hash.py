"""Chained block hashes of a token sequence, for the batched hash kernel's parity.

TEST INFRASTRUCTURE ONLY (like the rest of this package).

The nano vllm KV-cache practice page, section 4.2 ("前缀共享实现"), hashes a block
of tokens with h = (h * 31 + token) mod 2**32, seeded with the previous block's
hash, so the hash of full block b of a sequence covers its whole prefix. Written
out, that recursion is a polynomial in 31 over every token up to the end of the
block; this oracle evaluates that closed form directly with exact integers:

    H_b = sum_{i < e} t_i * 31**(e - 1 - i)  mod 2**32,   e = (b + 1) * block_size

(the seed of the first block is 0). Only full blocks are hashed.
"""
from __future__ import annotations

import numpy as np


def block_hashes(token_ids, block_size: int) -> np.ndarray:
    """uint32 [len(token_ids) // block_size]: the chained hash of each full block."""
    toks = [int(t) for t in token_ids]
    nb = len(toks) // int(block_size)
    out = np.zeros(nb, dtype=np.uint32)
    for b in range(nb):
        e = (b + 1) * block_size
        h = 0
        for i in range(e):
            h += toks[i] * pow(31, e - 1 - i)
        out[b] = h % (1 << 32)
    return out
