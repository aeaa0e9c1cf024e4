"""Pins on the input fixture: the rolling hash and the ref-counted block manager
(nano vllm KV-cache practice page, sections 3.2 and 4.2), and the generator."""
import os

import numpy as np
import pytest
import torch

from workloads import (CONFIGS, BlockManager, build_workload, compute_hash, f32_to_bf16_bits,
                       generate, relabel_blocks)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rolling_hash.txt")


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            prefix, toks, expect = (x.strip() for x in line.split(";"))
            rows.append((int(prefix), [int(t) for t in toks.split()], int(expect)))
    return rows


@pytest.mark.parametrize("prefix,toks,expect", _golden_rows())
def test_rolling_hash_golden(prefix, toks, expect):
    assert compute_hash(toks, prefix) == expect


def test_rolling_hash_chains_like_one_pass():
    # hashing two blocks chained == hashing their concatenation from the same seed
    a, b = [5, 9, 11, 2], [7, 7, 1, 3]
    assert compute_hash(b, compute_hash(a, 0)) == compute_hash(a + b, 0)


def test_block_manager_hit_miss_refcount_and_free():
    bm = BlockManager(8, 2, free_order=[3, 1, 4, 0, 5, 2, 7, 6])
    t1 = bm.allocate([1, 2, 3, 4, 5])        # blocks [1,2] [3,4] [5]
    assert t1 == [3, 1, 4]                    # taken in free-list order
    assert [bm.blocks[b].ref_count for b in t1] == [1, 1, 1]
    assert bm.blocks[3].hash == compute_hash([1, 2], 0)
    assert bm.blocks[1].hash == compute_hash([3, 4], compute_hash([1, 2], 0))
    assert bm.blocks[4].hash == -1            # partial block: not hashed
    t2 = bm.allocate([1, 2, 3, 4, 9, 9])     # shares the two full blocks, new third
    assert t2[:2] == [3, 1] and t2[2] == 0
    assert bm.blocks[3].ref_count == 2 and bm.blocks[1].ref_count == 2
    t3 = bm.allocate([1, 2, 8, 8])            # prefix diverges in the 2nd block
    assert t3[0] == 3 and t3[1] not in (1, 0, 4)
    assert bm.blocks[3].ref_count == 3
    bm.free_table(t1)
    assert bm.blocks[3].ref_count == 2 and bm.blocks[4].ref_count == 0
    bm.free_table(t2)
    bm.free_table(t3)
    assert bm.num_used() == 0
    assert all(b.hash == -1 for b in bm.blocks)
    with pytest.raises(RuntimeError):
        bm.free_table([3])


def test_block_manager_same_hash_different_tokens_not_shared():
    bm = BlockManager(4, 2)
    t1 = bm.allocate([1, 2])
    # force a colliding hash entry: a different chunk with the same hash value
    h = compute_hash([1, 2], 0)
    bm.hash_to_block_id[h] = t1[0]
    bm.blocks[t1[0]].token_ids = [9, 9]      # tokens no longer match
    t2 = bm.allocate([1, 2])
    assert t2[0] != t1[0]


def test_block_manager_partial_tail_reuses_cached_block():
    bm = BlockManager(8, 4)
    full = bm.allocate([1, 2, 3, 4, 5, 6, 7, 8])
    short = bm.allocate([1, 2, 3, 4, 5, 6])   # second block read partially
    assert short == full
    assert [bm.blocks[b].ref_count for b in full] == [2, 2]


def test_pool_exhaustion_raises():
    bm = BlockManager(2, 2)
    with pytest.raises(MemoryError):
        bm.allocate([1, 2, 3, 4, 5])


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 3,
                        np.array([1.0, -2.5, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 0.0, -0.0], np.float32)])
    ours = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_generator_is_deterministic_and_consistent():
    a = generate(CONFIGS["tiny_decode"])
    b = generate(CONFIGS["tiny_decode"])
    for f in ("context_lens", "block_tables", "q", "src_k", "src_v", "setup_slots", "new_slots"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert a.num_blocks == 256 and a.block_size == 16
    assert np.all((a.context_lens >= 1) & (a.context_lens <= 512))
    # every used physical block belongs to exactly one sequence (no sharing here)
    used = a.block_tables[a.block_tables >= 0]
    assert len(np.unique(used)) == len(used)
    assert used.max() < a.num_blocks
    # all slots distinct and inside the pool
    slots = np.concatenate([a.setup_slots, a.new_slots])
    assert len(np.unique(slots)) == len(slots)
    assert slots.min() >= 0 and slots.max() < a.num_blocks * a.block_size
    assert len(a.new_slots) == a.num_seqs      # one new token per sequence


def test_sharing_workload_refcounts_and_free():
    P, bs = 64, 16
    lens = np.array([10, 64, 100, 33, 200, 64, 17])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.zeros_like(lens),
                       num_q_heads=4, num_kv_heads=2, head_dim=8, block_size=bs, seed=3,
                       shared_prefix_len=P)
    nshared = P // bs
    shared_ids = None
    for s, L in enumerate(lens):
        k = -(-min(L, P) // bs)
        ids = w.block_tables[s, :k]
        if shared_ids is None or len(ids) > len(shared_ids):
            ref = shared_ids
            shared_ids = ids
            if ref is not None:
                assert np.array_equal(ids[:len(ref)], ref)
        else:
            assert np.array_equal(ids, shared_ids[:len(ids)])
    # ref_count(b-th shared block) = #{s : L_s > bs * b}
    for b in range(nshared):
        assert w.ref_counts[shared_ids[b]] == int(np.sum(lens > bs * b))
    # total references = sum over seqs of blocks used
    assert int(w.ref_counts.sum()) == int(sum(-(-int(L) // bs) for L in lens))
    # logical K of every sequence starts with the same shared rows
    k0 = w.logical_k(int(np.argmax(lens)))
    for s, L in enumerate(lens):
        m = min(int(L), P)
        assert np.array_equal(w.logical_k(s)[:m], k0[:m])
    # private-copy variant: same logical content, no block shared
    wp = build_workload(kind="decode", context_lens=lens, new_lens=np.zeros_like(lens),
                        num_q_heads=4, num_kv_heads=2, head_dim=8, block_size=bs, seed=3,
                        shared_prefix_len=P, share_prefix=False)
    used = wp.block_tables[wp.block_tables >= 0]
    assert len(np.unique(used)) == len(used)
    for s in range(len(lens)):
        assert np.array_equal(wp.logical_k(s), w.logical_k(s))


def test_prefix_share_config_saving_in_pages_range():
    """Config 4: unique vs logical bytes; the page reports 40-60% saving with shared
    prefixes (nano vllm page, section 3.2.2). The synthetic workload lands inside it."""
    w = generate(CONFIGS["prefix_share_decode"], num_seqs=128)
    saving = 1.0 - w.kv_bytes_unique() / w.kv_bytes_logical()
    assert 0.3 < saving < 0.7


def test_relabel_blocks_moves_slots_with_tables():
    w = generate(CONFIGS["tiny_decode"])
    perm = np.random.default_rng(1).permutation(w.num_blocks)
    r = relabel_blocks(w, perm)
    bs = w.block_size
    for s in range(w.num_seqs):
        for p in range(int(w.context_lens[s])):
            a = int(w.block_tables[s, p // bs]) * bs + p % bs
            b = int(r.block_tables[s, p // bs]) * bs + p % bs
            assert b == perm[a // bs] * bs + a % bs


def test_block_manager_append_fresh_private_and_shared():
    bm = BlockManager(num_blocks=8, block_size=2, free_order=[3, 1, 4, 0, 5, 2, 6, 7])
    a = bm.allocate([1, 2, 3])              # blocks 3 (full, hashed), 1 (partial)
    slot, cp = bm.append(a, 3, 9)            # into the private partial block 1
    assert (slot, cp) == (1 * 2 + 1, None) and bm.blocks[1].token_ids == [3, 9]
    slot, cp = bm.append(a, 4, 5)            # starts a block: fresh block 4
    assert (slot, cp) == (4 * 2, None) and a == [3, 1, 4]
    b = bm.allocate([1, 2, 7])               # shares block 3 with a
    assert b[0] == 3 and bm.blocks[3].ref_count == 2
    # a second request whose partial tail reuses a cached full block, then appends to it
    c = bm.allocate([1])                     # partial tail [1] is a prefix of block 3's tokens
    assert c == [3] and bm.blocks[3].ref_count == 3
    slot, cp = bm.append(c, 1, 8)            # shared: copy-on-write into a fresh block
    assert cp == (3, c[0]) and c[0] != 3 and slot == c[0] * 2 + 1
    assert bm.blocks[3].ref_count == 2 and bm.blocks[c[0]].token_ids == [1, 8]
    assert bm.blocks[3].token_ids == [1, 2]  # the shared block is untouched


def test_block_manager_append_into_private_hashed_block_forgets_its_hash():
    bm = BlockManager(num_blocks=4, block_size=2)
    a = bm.allocate([1, 2])                  # block 0, hashed
    bm.free_table(a)                         # freed: hash forgotten, back on the free list
    c = bm.allocate([1, 2])                  # block 1 (the free list continues), hashed
    h = bm.blocks[c[0]].hash
    d = bm.allocate([1])                     # partial tail reuses block c[0]
    bm.free_table(c)                         # c finishes: d holds the block alone
    assert bm.blocks[d[0]].ref_count == 1 and bm.blocks[d[0]].hash == h
    slot, cp = bm.append(d, 1, 5)            # private but hashed: forget, write in place
    assert cp is None and slot == d[0] * 2 + 1
    assert bm.blocks[d[0]].hash == -1 and h not in bm.hash_to_block_id
    assert bm.blocks[d[0]].token_ids == [1, 5]
