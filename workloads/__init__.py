"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

Holds no attention arithmetic: lengths, values, token ids, block allocation and
the slots rows must be written to.
"""
from .block_manager import Block, BlockManager, compute_hash
from .configs import CONFIGS, WorkloadConfig
from .gen import (SENTINEL_BF16, Workload, build_workload, copy_on_write_append, f32_to_bf16_bits,
                  generate, relabel_blocks)

__all__ = ["Block", "BlockManager", "compute_hash", "CONFIGS", "WorkloadConfig", "SENTINEL_BF16",
           "Workload", "build_workload", "copy_on_write_append", "f32_to_bf16_bits", "generate",
           "relabel_blocks"]
