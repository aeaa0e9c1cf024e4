"""Helpers shared by the GPU parity tests: move a seeded workload to the device,
run the library through its Python binding, and run the oracle on the same bits."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_442_b200 as pa
from workloads import SENTINEL_BF16

# Parity bar ("max abs error 1e-2 with relative error 1e-2 on bf16 outputs"):
#   per element |g - r| <= TOL_ABS + TOL_REL * |r|   (the abs+rel "allclose" form: a
#     bf16 output of magnitude >= 4 is already up to 2**-6 = 0.0156 away from the exact
#     value after its one mandated rounding, so a bare 1e-2 absolute bound would reject
#     correctly rounded results), and
#   over the whole tensor ||g - r||_2 / ||r||_2 <= TOL_NORM (keeps the check meaningful
#     at long context, where outputs are ~1e-2 and the element bound alone is loose).
TOL_ABS = 1e-2
TOL_REL = 1e-2
TOL_NORM = 1e-2


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bf16 tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def i32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class DeviceWorkload:
    """A workload's pools and metadata on the GPU; setup rows already stored."""

    def __init__(self, w, store_new: bool = True):
        self.w = w
        shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
        fill = torch.tensor(SENTINEL_BF16, dtype=torch.int32).to(torch.int16)
        self.k_cache = torch.full(shape, int(fill), dtype=torch.int16, device="cuda").view(torch.bfloat16)
        self.v_cache = torch.full(shape, int(fill), dtype=torch.int16, device="cuda").view(torch.bfloat16)
        self.block_tables = i32_dev(w.block_tables)
        self.context_lens = i32_dev(w.context_lens)
        self.cu_seqlens_q = i32_dev(w.cu_seqlens_q)
        self.q = bf16_dev(w.q)
        if len(w.setup_slots):
            pa.pa_store_kvcache(bf16_dev(w.setup_k), bf16_dev(w.setup_v), self.k_cache,
                                self.v_cache, i32_dev(w.setup_slots))
        self.new_k = bf16_dev(w.new_k) if len(w.new_slots) else None
        self.new_v = bf16_dev(w.new_v) if len(w.new_slots) else None
        self.new_slots = i32_dev(w.new_slots)
        if store_new:
            self.store_new()

    def store_new(self):
        if self.new_k is not None:
            pa.pa_store_kvcache(self.new_k, self.new_v, self.k_cache, self.v_cache, self.new_slots)

    def decode(self, partition_size: int = 0, q=None) -> torch.Tensor:
        w = self.w
        q = self.q if q is None else q
        out = torch.empty_like(q)
        ws, P = pa.decode_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                    w.max_context_len, partition_size)
        pa.pa_decode(out, q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                     w.scale, w.max_context_len, P, ws)
        return out

    def prefill(self) -> torch.Tensor:
        w = self.w
        out = torch.empty_like(self.q)
        max_q = int(np.max(np.diff(w.cu_seqlens_q))) if w.num_seqs else 0
        pa.pa_prefill(out, self.q, self.k_cache, self.v_cache, self.block_tables,
                      self.cu_seqlens_q, self.context_lens, w.scale, max_q)
        return out


def oracle_pools(w):
    kc, vc = w.empty_pool(), w.empty_pool()
    if len(w.setup_slots):
        kc, vc = oracle.store_kvcache(kc, vc, w.setup_k, w.setup_v, w.setup_slots)
    if len(w.new_slots):
        kc, vc = oracle.store_kvcache(kc, vc, w.new_k, w.new_v, w.new_slots)
    return kc, vc


def oracle_decode(w, pools=None, seqs=None):
    kc, vc = pools if pools is not None else oracle_pools(w)
    if seqs is None:
        return oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
    seqs = np.asarray(seqs)
    return oracle.decode(w.q[seqs], kc, vc, w.block_tables[seqs], w.context_lens[seqs], w.scale)


def oracle_prefill(w, pools=None):
    kc, vc = pools if pools is not None else oracle_pools(w)
    return oracle.prefill(w.q, kc, vc, w.block_tables, w.cu_seqlens_q, w.context_lens, w.scale)


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    c = oracle.compare(gpu, ref)
    assert c["finite"], f"{what}: non-finite GPU output"
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    excess = np.abs(g - r) - (TOL_ABS + TOL_REL * np.abs(r))
    c["worst_excess"] = float(excess.max()) if excess.size else 0.0
    assert c["worst_excess"] <= 0.0 and c["norm_rel"] <= TOL_NORM, f"{what}: {c}"
    return c
