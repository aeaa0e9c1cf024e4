"""The five synthetic workloads the paged-attention path is tested and measured on.

Shapes follow the engine configuration printed on the nano vllm KV-cache practice
page (section 2.2: 16384 batched tokens, 512 sequences, 4096 maximum length, block
size 256) and the mini-vllm page's block-table KV cache (section 2, "KVCache").
Where the pages leave a number open, the value here is a stated reading: the
lognormal spread (sigma 1), the pool size (10% spare), the seeds and which
positions are stored inside the measured step.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

SEED_BASE = 20261202


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    index: int               # 1..5, also selects the seed
    kind: str                # "decode" or "prefill"
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    # decode: context length distribution (inclusive bounds / lognormal params)
    ctx_dist: str = "uniform"          # "uniform" | "fixed" | "lognormal"
    ctx_lo: int = 1
    ctx_hi: int = 1
    lognormal_median: float = 1024.0
    lognormal_sigma: float = 1.0
    # pool: fixed size, or None -> ceil(1.1 * blocks needed)
    pool_blocks: int | None = None
    # decode: store the last position of each sequence inside the step
    store_new_tokens: bool = True
    # prefix sharing: positions < shared_prefix_len map to shared blocks
    shared_prefix_len: int = 0
    # prefill: cached prefix length and new tokens per sequence
    prefix_len: int = 0
    new_tokens: int = 0

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def max_context_len(self) -> int:
        if self.kind == "prefill":
            return self.prefix_len + self.new_tokens
        return self.ctx_hi


TINY_DECODE = WorkloadConfig(
    name="tiny_decode", index=1, kind="decode", num_seqs=4, num_q_heads=8, num_kv_heads=8,
    head_dim=64, block_size=16, ctx_dist="uniform", ctx_lo=1, ctx_hi=512, pool_blocks=256,
    store_new_tokens=True)

DECODE_B64 = WorkloadConfig(
    name="decode_b64", index=2, kind="decode", num_seqs=64, num_q_heads=16, num_kv_heads=8,
    head_dim=128, block_size=256, ctx_dist="uniform", ctx_lo=512, ctx_hi=4096,
    store_new_tokens=True)

LONG_CTX_DECODE = WorkloadConfig(
    name="long_ctx_decode", index=3, kind="decode", num_seqs=8, num_q_heads=32, num_kv_heads=8,
    head_dim=128, block_size=256, ctx_dist="fixed", ctx_lo=32768, ctx_hi=32768,
    store_new_tokens=True)

PREFIX_SHARE_DECODE = WorkloadConfig(
    name="prefix_share_decode", index=4, kind="decode", num_seqs=512, num_q_heads=32,
    num_kv_heads=8, head_dim=128, block_size=64, ctx_dist="lognormal", ctx_lo=1, ctx_hi=4096,
    lognormal_median=1024.0, lognormal_sigma=1.0, store_new_tokens=False,
    shared_prefix_len=1024)

CHUNKED_PREFILL = WorkloadConfig(
    name="chunked_prefill", index=5, kind="prefill", num_seqs=32, num_q_heads=32,
    num_kv_heads=8, head_dim=128, block_size=256, prefix_len=2048, new_tokens=512)

CONFIGS = {c.name: c for c in (TINY_DECODE, DECODE_B64, LONG_CTX_DECODE,
                               PREFIX_SHARE_DECODE, CHUNKED_PREFILL)}
