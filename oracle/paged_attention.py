"""Plain CPU oracle of the paged KV-cache hot path: store, block-table gather,
decode attention and causal chunked prefill, in float64.

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports this module;
only the tests, the smoke check and the benchmark's CPU-baseline leg may call it.
It shares no code with the CUDA path.

What it follows:
  * fixed-size blocks, each holding the K/V of a run of consecutive token
    positions, stored non-contiguously in a pre-allocated pool (nano vllm
    KV-cache practice page, section 3.2.1; mini-vllm page, "PagedAttention 核心思想");
  * a per-sequence block table decides where in the pre-allocated tensor each
    position's K/V is read and written (nano vllm page, section 3.1, the
    Sequence's block_table; mini-vllm page, section 2 "KVCache");
  * during decode one query token per sequence attends over everything cached so
    far (mini-vllm page, "性能评估与基准测试"): the result must equal recomputing
    attention over the whole sequence, which is what this oracle literally does.

The attention itself is the textbook definition: z_j = scale * (q . k_j),
w = softmax(z) (subtract the max, exponentiate, normalise), out = sum_j w_j v_j.
Readings fixed by this implementation (the pages give none of them):
  * pool layout [num_blocks, block_size, num_kv_heads, head_dim]; the row of
    logical position p of a sequence is block_table[p // block_size] *
    block_size + p % block_size;
  * grouped-query attention: query head h reads kv head h // (Hq / Hkv);
  * decode: context_lens includes the token being decoded, whose K/V has already
    been stored; no mask beyond the context length;
  * prefill: new token i of a sequence with n_new new tokens sits at absolute
    position ctx - n_new + i and sees positions 0..pos (causal);
  * a sequence with context length <= 0 produces an all-zero output row.

bf16 values travel as uint16 bit patterns; every bf16 value is exactly
representable in float64, so the oracle reads exactly the bits the GPU reads.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact conversion of bf16 bit patterns (uint16) to float64."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# a1: write new K/V rows into the pool through the slot mapping
# ---------------------------------------------------------------------------
def store_kvcache(k_cache: np.ndarray, v_cache: np.ndarray, k: np.ndarray, v: np.ndarray,
                  slot_mapping: np.ndarray):
    """Return copies of the pools with row slot_mapping[t] replaced by k[t] / v[t].

    k_cache, v_cache: uint16 [num_blocks, block_size, Hkv, D]; k, v: uint16
    [T, Hkv, D]; slot_mapping: int [T], a negative slot means "skip this token".
    Rows that no token targets keep their previous bytes.
    """
    kc = np.array(k_cache, dtype=np.uint16, copy=True)
    vc = np.array(v_cache, dtype=np.uint16, copy=True)
    nb, bs, hkv, d = kc.shape
    kflat = kc.reshape(nb * bs, hkv, d)
    vflat = vc.reshape(nb * bs, hkv, d)
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        if slot >= nb * bs:
            raise IndexError(f"slot {slot} outside a pool of {nb * bs} rows")
        kflat[slot] = k[t]
        vflat[slot] = v[t]
    return kc, vc


# ---------------------------------------------------------------------------
# copy-on-write: a private copy of a shared block before a sequence appends to it
# ---------------------------------------------------------------------------
def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, src_blocks: np.ndarray,
                dst_blocks: np.ndarray):
    """Return copies of the pools in which block dst_blocks[i] holds what block
    src_blocks[i] held, in K and in V.

    Blocks are shared between sequences by reference count (nano vllm page, section
    3.2.1); the page does not say what happens when a sequence writes into a shared
    block. Reading taken: the writer first gets a private copy (copy-on-write), so
    the other sharers keep reading the unchanged block. Every source is read before
    any destination is written; destinations must be distinct and must not also be
    sources of the same call.
    """
    kc = np.array(k_cache, dtype=np.uint16, copy=True)
    vc = np.array(v_cache, dtype=np.uint16, copy=True)
    src = [int(b) for b in src_blocks]
    dst = [int(b) for b in dst_blocks]
    nb = kc.shape[0]
    if len(src) != len(dst):
        raise ValueError("src_blocks and dst_blocks differ in length")
    if any(b < 0 or b >= nb for b in src + dst):
        raise IndexError("block id outside the pool")
    if len(set(dst)) != len(dst) or set(dst) & set(src):
        raise ValueError("destinations must be distinct and not also sources")
    for a, b in zip(src, dst):
        kc[b] = k_cache[a]
        vc[b] = v_cache[a]
    return kc, vc


# ---------------------------------------------------------------------------
# a2: logical position -> pool row, and the gather of one sequence
# ---------------------------------------------------------------------------
def physical_row(block_table_row: np.ndarray, pos: int, block_size: int) -> int:
    """Pool row holding logical position `pos` of a sequence."""
    block = int(block_table_row[pos // block_size])
    if block < 0:
        raise IndexError(f"position {pos} falls in an unallocated block")
    return block * block_size + pos % block_size


def gather_sequence(cache: np.ndarray, block_table_row: np.ndarray, length: int) -> np.ndarray:
    """Contiguous [length, Hkv, D] copy of a sequence's first `length` positions."""
    nb, bs, hkv, d = cache.shape
    flat = cache.reshape(nb * bs, hkv, d)
    rows = [physical_row(block_table_row, p, bs) for p in range(length)]
    return flat[np.asarray(rows, dtype=np.int64)] if rows else np.zeros((0, hkv, d), cache.dtype)


# ---------------------------------------------------------------------------
# textbook softmax attention of one query against n keys
# ---------------------------------------------------------------------------
def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """q [D], K [n, D], V [n, D] (float64) -> [D]; zeros when n == 0."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    z = scale * (K @ q)
    z = z - z.max()
    w = np.exp(z)
    w = w / w.sum()
    return w @ V


# ---------------------------------------------------------------------------
# a3 + a4: decode (one query token per sequence)
# ---------------------------------------------------------------------------
def decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_tables: np.ndarray,
           context_lens: np.ndarray, scale: float) -> np.ndarray:
    """Paged decode attention; returns float64 [B, Hq, D].

    q: uint16 bf16 bits [B, Hq, D]; caches: uint16 [num_blocks, bs, Hkv, D];
    block_tables: int [B, max_blocks]; context_lens: int [B].
    """
    B, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    G = Hq // Hkv
    scale = float(np.float32(scale))
    qf = bf16_bits_to_f64(q)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for s in range(B):
        ctx = int(context_lens[s])
        if ctx <= 0:
            continue
        Kc = bf16_bits_to_f64(gather_sequence(k_cache, block_tables[s], ctx))
        Vc = bf16_bits_to_f64(gather_sequence(v_cache, block_tables[s], ctx))
        for h in range(Hq):
            g = h // G
            out[s, h] = softmax_attention(qf[s, h], Kc[:, g, :], Vc[:, g, :], scale)
    return out


# ---------------------------------------------------------------------------
# a5: causal chunked prefill onto a cached prefix
# ---------------------------------------------------------------------------
def prefill(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_tables: np.ndarray,
            cu_seqlens_q: np.ndarray, context_lens: np.ndarray, scale: float) -> np.ndarray:
    """Causal paged prefill; returns float64 [total_new, Hq, D].

    Sequence s owns query rows cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1; its K/V
    (prefix and the new tokens, already stored) live in the pool.
    """
    Tq, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    G = Hq // Hkv
    scale = float(np.float32(scale))
    qf = bf16_bits_to_f64(q)
    out = np.zeros((Tq, Hq, D), dtype=np.float64)
    B = len(context_lens)
    for s in range(B):
        q0, q1 = int(cu_seqlens_q[s]), int(cu_seqlens_q[s + 1])
        n_new = q1 - q0
        ctx = int(context_lens[s])
        if n_new <= 0 or ctx <= 0:
            continue
        if n_new > ctx:
            raise ValueError("a sequence cannot have more new tokens than context")
        first = ctx - n_new
        Kc = bf16_bits_to_f64(gather_sequence(k_cache, block_tables[s], ctx))
        Vc = bf16_bits_to_f64(gather_sequence(v_cache, block_tables[s], ctx))
        pos = first + np.arange(n_new)
        visible = np.arange(ctx)[None, :] <= pos[:, None]          # [n_new, ctx]
        for h in range(Hq):
            g = h // G
            Z = scale * (qf[q0:q1, h, :] @ Kc[:, g, :].T)              # [n_new, ctx]
            Z = np.where(visible, Z, -np.inf)
            Z = Z - Z.max(axis=1, keepdims=True)
            W = np.exp(Z)
            W = W / W.sum(axis=1, keepdims=True)
            out[q0:q1, h, :] = W @ Vc[:, g, :]
    return out


# ---------------------------------------------------------------------------
# comparison used by every parity check
# ---------------------------------------------------------------------------
def compare(gpu: np.ndarray, ref: np.ndarray) -> dict:
    """max |g - r| and ||g - r||_2 / ||r||_2 over a whole output tensor."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    diff = g - r
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    rn = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(diff) / rn) if rn > 0 else float(np.linalg.norm(diff))
    return {"max_abs": max_abs, "norm_rel": rel, "finite": bool(np.all(np.isfinite(g)))}
