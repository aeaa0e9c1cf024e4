"""Seeded synthetic inputs for the paged KV cache (both the CUDA path and the oracle).

This module holds no attention arithmetic. It draws context lengths, K/V/q values
and token ids, asks the block manager for block tables, and turns (sequence,
position) into the pool slot the row has to be written to. Everything is numpy on
the CPU; bf16 values are carried as their uint16 bit patterns.

Recipe (one numpy PCG64 stream per purpose, spawned from the workload's seed):
  * lengths: uniform (inclusive bounds), fixed, or
    clip(rint(exp(N(ln median, sigma))), 1, max);
  * values: float32 N(0, 1) rounded once, to nearest even, to bf16; q optionally
    multiplied by a factor before rounding (the "peaked" variant);
  * token ids: uniform in [1, 2**31 - 1]; the shared prefix of the sharing
    workload uses one id list for every sequence;
  * physical block ids: the block manager's free list is a seeded permutation of
    the pool, so consecutive logical blocks land on scattered physical blocks.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from .block_manager import BlockManager
from .configs import WorkloadConfig

SENTINEL_BF16 = 0xFFC1  # a quiet-NaN bf16 pattern that unwritten pool rows hold


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits.

    Inputs are finite draws, so no NaN/Inf handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def _normal_bf16(rng: np.random.Generator, shape, factor: float = 1.0, chunk: int = 1 << 24):
    """Draw float32 N(0,1) of `shape`, scale, round to bf16 bits (chunked for memory)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = rng.standard_normal(e - s, dtype=np.float32)
        if factor != 1.0:
            x *= np.float32(factor)
        out[s:e] = f32_to_bf16_bits(x)
    return out.reshape(shape)


@dataclass
class Workload:
    """Everything one call of the paged path needs, plus bookkeeping for the tests."""

    kind: str                      # "decode" | "prefill"
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float                   # float32-representable
    context_lens: np.ndarray       # int32 [B], includes this step's new tokens
    new_lens: np.ndarray           # int32 [B], positions ctx-new .. ctx-1 are stored in the step
    block_tables: np.ndarray       # int32 [B, max_blocks], -1 padded
    q: np.ndarray                  # uint16 bf16 bits: decode [B,Hq,D]; prefill [sum(new),Hq,D]
    cu_seqlens_q: np.ndarray       # int32 [B+1] (prefill query offsets; decode: arange)
    src_k: np.ndarray              # uint16 [R, Hkv, D] distinct source rows
    src_v: np.ndarray
    logical_rows: list             # per seq: int64 [ctx] index into src rows, by position
    setup_slots: np.ndarray        # int32 [Ns] slots written before the step
    setup_src: np.ndarray          # int64 [Ns] source row per setup slot
    new_slots: np.ndarray          # int32 [Tn] slots written inside the step
    new_src: np.ndarray            # int64 [Tn]
    ref_counts: np.ndarray = field(default=None)  # int32 [num_blocks] after allocation
    name: str = "custom"

    # convenience views -------------------------------------------------------
    @property
    def setup_k(self):
        return self.src_k[self.setup_src]

    @property
    def setup_v(self):
        return self.src_v[self.setup_src]

    @property
    def new_k(self):
        return self.src_k[self.new_src]

    @property
    def new_v(self):
        return self.src_v[self.new_src]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    def logical_k(self, s: int) -> np.ndarray:
        """Contiguous [ctx, Hkv, D] K of sequence s, by construction (no block table)."""
        return self.src_k[self.logical_rows[s]]

    def logical_v(self, s: int) -> np.ndarray:
        return self.src_v[self.logical_rows[s]]

    def empty_pool(self) -> np.ndarray:
        """One pool (K or V) filled with the sentinel bit pattern."""
        return np.full((self.num_blocks, self.block_size, self.num_kv_heads, self.head_dim),
                       SENTINEL_BF16, dtype=np.uint16)

    def kv_bytes_logical(self) -> int:
        """K+V bytes a decode reads when every logical position is read once."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_dim * 2 * 2

    def kv_bytes_unique(self) -> int:
        """K+V bytes of the distinct (slot) rows the sequences touch."""
        slots = set()
        bs = self.block_size
        for s in range(self.num_seqs):
            ctx = int(self.context_lens[s])
            nb = -(-ctx // bs)
            for b in range(nb):
                rows = min(bs, ctx - b * bs)
                base = int(self.block_tables[s, b]) * bs
                slots.update(range(base, base + rows))
        return len(slots) * self.num_kv_heads * self.head_dim * 2 * 2


def _lengths(cfg: WorkloadConfig, rng: np.random.Generator) -> np.ndarray:
    B = cfg.num_seqs
    if cfg.kind == "prefill":
        return np.full(B, cfg.prefix_len + cfg.new_tokens, dtype=np.int64)
    if cfg.ctx_dist == "uniform":
        return rng.integers(cfg.ctx_lo, cfg.ctx_hi, size=B, endpoint=True).astype(np.int64)
    if cfg.ctx_dist == "fixed":
        return np.full(B, cfg.ctx_lo, dtype=np.int64)
    if cfg.ctx_dist == "lognormal":
        z = rng.normal(math.log(cfg.lognormal_median), cfg.lognormal_sigma, size=B)
        return np.clip(np.rint(np.exp(z)), cfg.ctx_lo, cfg.ctx_hi).astype(np.int64)
    raise ValueError(cfg.ctx_dist)


def build_workload(*, kind: str, context_lens, new_lens, num_q_heads: int, num_kv_heads: int,
                   head_dim: int, block_size: int, seed: int, pool_blocks: int | None = None,
                   shared_prefix_len: int = 0, share_prefix: bool = True, q_factor: float = 1.0,
                   name: str = "custom") -> Workload:
    """Build a workload from explicit per-sequence lengths.

    context_lens[s]: total tokens of sequence s after this step's writes;
    new_lens[s]: how many of its last positions are written inside the step (decode:
    0 or 1; prefill: the number of new query tokens).
    """
    ctx = np.asarray(context_lens, dtype=np.int64)
    new = np.asarray(new_lens, dtype=np.int64)
    B = int(ctx.shape[0])
    if new.shape != ctx.shape or np.any(new < 0) or np.any(new > ctx):
        raise ValueError("need 0 <= new_lens <= context_lens")
    if kind == "decode" and np.any(new > 1):
        raise ValueError("a decode step writes at most one token per sequence")
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    ss = np.random.SeedSequence(seed)
    rng_data, rng_tok, rng_perm = (np.random.default_rng(c) for c in ss.spawn(3))
    Hkv, D, bs = num_kv_heads, head_dim, block_size

    # -- logical source rows ------------------------------------------------
    P = int(shared_prefix_len)
    own = np.maximum(ctx - P, 0) if P else ctx.copy()
    n_src = (P if P else 0) + int(own.sum())
    src_k = _normal_bf16(rng_data, (n_src, Hkv, D))
    src_v = _normal_bf16(rng_data, (n_src, Hkv, D))
    logical_rows = []
    base = P
    for s in range(B):
        c = int(ctx[s])
        if P:
            shared = np.arange(min(c, P), dtype=np.int64)
            mine = np.arange(base, base + max(c - P, 0), dtype=np.int64)
            base += max(c - P, 0)
            logical_rows.append(np.concatenate([shared, mine]))
        else:
            logical_rows.append(np.arange(base, base + c, dtype=np.int64))
            base += c
    # -- queries -------------------------------------------------------------
    if kind == "decode":
        q = _normal_bf16(rng_data, (B, num_q_heads, D), factor=q_factor)
        cu = np.arange(B + 1, dtype=np.int32)
    elif kind == "prefill":
        q = _normal_bf16(rng_data, (int(new.sum()), num_q_heads, D), factor=q_factor)
        cu = np.zeros(B + 1, dtype=np.int32)
        cu[1:] = np.cumsum(new)
    else:
        raise ValueError(kind)

    # -- token ids and block allocation ---------------------------------------
    hi = 2 ** 31 - 1
    prefix_ids = rng_tok.integers(1, hi, size=P) if P else None
    token_lists = []
    for s in range(B):
        c = int(ctx[s])
        if P and share_prefix:
            head = prefix_ids[:min(c, P)]
        elif P:
            head = rng_tok.integers(1, hi, size=min(c, P))
        else:
            head = np.zeros(0, dtype=np.int64)
        tail = rng_tok.integers(1, hi, size=max(c - P, 0) if P else c)
        token_lists.append(np.concatenate([head, tail]).tolist())

    def allocate(num_blocks, order):
        bm = BlockManager(num_blocks, bs, order)
        system = bm.allocate(prefix_ids.tolist()) if (P and share_prefix) else None
        tables = [bm.allocate(t) for t in token_lists]
        if system is not None:
            bm.free_table(system)  # the system prompt request finishes; its blocks stay shared
        return bm, tables

    if pool_blocks is None:
        total_logical = int(sum(-(-int(c) // bs) for c in ctx)) + (-(-P // bs) if P else 0)
        bm0, _ = allocate(max(total_logical, 1), None)
        used = bm0.num_used()
        num_blocks = max(1, math.ceil(1.1 * used))
    else:
        num_blocks = int(pool_blocks)
    perm = rng_perm.permutation(num_blocks)
    bm, tables = allocate(num_blocks, perm)
    max_blocks = max([len(t) for t in tables] + [1])
    block_tables = np.full((B, max_blocks), -1, dtype=np.int32)
    for s, t in enumerate(tables):
        block_tables[s, :len(t)] = t

    # -- slots: (seq, position) -> pool row -------------------------------------
    setup = {}
    new_slots, new_src = [], []
    for s in range(B):
        c = int(ctx[s])
        first_new = c - int(new[s])
        rows = logical_rows[s]
        for p in range(c):
            slot = int(block_tables[s, p // bs]) * bs + p % bs
            if p >= first_new:
                new_slots.append(slot)
                new_src.append(int(rows[p]))
            else:
                prev = setup.get(slot)
                if prev is not None and prev != int(rows[p]):
                    raise AssertionError("two different rows mapped to one shared slot")
                setup[slot] = int(rows[p])
    setup_slots = np.fromiter(setup.keys(), dtype=np.int32, count=len(setup))
    setup_src = np.fromiter(setup.values(), dtype=np.int64, count=len(setup))

    return Workload(
        kind=kind, num_seqs=B, num_q_heads=num_q_heads, num_kv_heads=Hkv, head_dim=D,
        block_size=bs, num_blocks=num_blocks, scale=float(np.float32(1.0 / math.sqrt(D))),
        context_lens=ctx.astype(np.int32), new_lens=new.astype(np.int32),
        block_tables=block_tables, q=q, cu_seqlens_q=cu, src_k=src_k, src_v=src_v,
        logical_rows=logical_rows, setup_slots=setup_slots, setup_src=setup_src,
        new_slots=np.asarray(new_slots, dtype=np.int32), new_src=np.asarray(new_src, dtype=np.int64),
        ref_counts=np.asarray(bm.ref_counts(), dtype=np.int32), name=name)


def generate(cfg: WorkloadConfig, *, q_factor: float = 1.0, share_prefix: bool = True,
             num_seqs: int | None = None) -> Workload:
    """The seeded workload of one named configuration.

    num_seqs, when given, keeps only the first sequences of the drawn lengths (a
    deterministic subset used for bounded CPU timing and sampled checks).
    """
    ss = np.random.SeedSequence(cfg.seed)
    rng_len = np.random.default_rng(ss.spawn(1)[0])
    lens = _lengths(cfg, rng_len)
    if num_seqs is not None:
        lens = lens[:num_seqs]
    if cfg.kind == "prefill":
        new = np.full(lens.shape, cfg.new_tokens, dtype=np.int64)
    else:
        new = np.where(lens > 0, 1 if cfg.store_new_tokens else 0, 0)
    return build_workload(kind=cfg.kind, context_lens=lens, new_lens=new,
                          num_q_heads=cfg.num_q_heads, num_kv_heads=cfg.num_kv_heads,
                          head_dim=cfg.head_dim, block_size=cfg.block_size, seed=cfg.seed + 1000,
                          pool_blocks=cfg.pool_blocks, shared_prefix_len=cfg.shared_prefix_len,
                          share_prefix=share_prefix, q_factor=q_factor, name=cfg.name)


def copy_on_write_append(w: Workload):
    """A decode step in which every sequence appends (stores) its last position into a
    block no other sequence of the batch reads.

    With shared prefixes the last position of a short sequence can fall in a block
    other sequences also read (reference count > 1; nano vllm page, section 3.2.1).
    Such a block is first copied to a fresh physical block that only this sequence's
    table points at; the last sharer to append keeps the original. New blocks are
    appended to the pool (ids num_blocks, num_blocks + 1, ...). This is host-side
    block management: which blocks to copy, and the resulting tables and slots.

    Returns (workload whose step stores the last row of every sequence,
             src_blocks int32 [n], dst_blocks int32 [n]).
    """
    bs = w.block_size
    refs = np.zeros(w.num_blocks, dtype=np.int64)
    for s in range(w.num_seqs):
        n = -(-int(w.context_lens[s]) // bs)
        for b in w.block_tables[s, :n]:
            refs[int(b)] += 1
    bt = w.block_tables.copy()
    src, dst, new_slots, new_src = [], [], [], []
    nxt = w.num_blocks
    for s in range(w.num_seqs):
        ctx = int(w.context_lens[s])
        if ctx <= 0:
            continue
        last = ctx - 1
        bi = last // bs
        b = int(bt[s, bi])
        if refs[b] > 1:
            src.append(b)
            dst.append(nxt)
            refs[b] -= 1
            bt[s, bi] = nxt
            nxt += 1
        new_slots.append(int(bt[s, bi]) * bs + last % bs)
        new_src.append(int(w.logical_rows[s][last]))
    rc = np.concatenate([refs, np.ones(nxt - w.num_blocks, dtype=np.int64)]).astype(np.int32)
    w2 = Workload(**{**w.__dict__, "num_blocks": nxt, "block_tables": bt,
                     "new_lens": (w.context_lens > 0).astype(np.int32),
                     "new_slots": np.asarray(new_slots, dtype=np.int32),
                     "new_src": np.asarray(new_src, dtype=np.int64), "ref_counts": rc,
                     "name": w.name + "+cow"})
    return w2, np.asarray(src, dtype=np.int32), np.asarray(dst, dtype=np.int32)


def relabel_blocks(w: Workload, perm: np.ndarray) -> Workload:
    """Same logical content with physical block b renamed perm[b] (tables and slots)."""
    perm = np.asarray(perm, dtype=np.int64)
    if sorted(perm.tolist()) != list(range(w.num_blocks)):
        raise ValueError("perm must be a permutation of the pool")
    bs = w.block_size

    def map_slots(slots):
        slots = slots.astype(np.int64)
        return (perm[slots // bs] * bs + slots % bs).astype(np.int32)

    bt = w.block_tables.astype(np.int64)
    bt = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    rc = np.zeros_like(w.ref_counts)
    rc[perm] = w.ref_counts
    return Workload(**{**w.__dict__, "block_tables": bt,
                       "setup_slots": map_slots(w.setup_slots),
                       "new_slots": map_slots(w.new_slots), "ref_counts": rc})
