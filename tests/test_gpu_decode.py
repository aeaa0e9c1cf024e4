"""GPU parity of store_kvcache and paged decode against the CPU oracle.

Bar: store and block indexing bit-exact; decode outputs within
|g-r| <= 1e-2 + 1e-2 |r| per element and ||g-r||/||r|| <= 1e-2 of the fp64 oracle
on the same seeded bf16 inputs.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import (DeviceWorkload, assert_close, bf16_dev, i32_dev, oracle_decode,
                               oracle_pools, to_bits, to_f64)
from workloads import CONFIGS, build_workload, generate, relabel_blocks

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ store
@pytest.mark.parametrize("name", ["tiny_decode", "decode_b64"])
def test_store_pool_bytes_bit_exact(name):
    w = generate(CONFIGS[name])
    dw = DeviceWorkload(w)
    kc, vc = oracle_pools(w)
    torch.cuda.synchronize()
    assert np.array_equal(to_bits(dw.k_cache), kc)
    assert np.array_equal(to_bits(dw.v_cache), vc)


def test_store_16k_prefill_tokens_bit_exact():
    w = generate(CONFIGS["chunked_prefill"], num_seqs=32)
    dw = DeviceWorkload(w)
    kc, vc = oracle_pools(w)
    assert np.array_equal(to_bits(dw.k_cache), kc)
    assert np.array_equal(to_bits(dw.v_cache), vc)


def test_store_skips_negative_slots_and_flags_bad_ones():
    w = generate(CONFIGS["tiny_decode"])
    dw = DeviceWorkload(w, store_new=False)
    before_k = to_bits(dw.k_cache).copy()
    slots = w.new_slots.copy()
    slots[0] = -1
    pa.pa_store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, i32_dev(slots))
    after = to_bits(dw.k_cache).reshape(-1, w.num_kv_heads, w.head_dim)
    flat_before = before_k.reshape(-1, w.num_kv_heads, w.head_dim)
    assert np.array_equal(after[w.new_slots[0]], flat_before[w.new_slots[0]])
    for t in range(1, len(slots)):
        assert np.array_equal(after[slots[t]], w.new_k[t])
    # a slot past the pool: skipped, reported as a bad index in debug mode, no fault
    bad = slots.copy()
    bad[1] = w.num_blocks * w.block_size + 5
    pa.pa_set_debug_checks(True)
    try:
        with pytest.raises(pa.PAError) as e:
            pa.pa_store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, i32_dev(bad))
        assert e.value.status == 3
    finally:
        pa.pa_set_debug_checks(True)
    assert pa.pa_check_device_errors() == 0


def test_gather_reconstructs_every_sequence_bit_exact():
    """Reading each sequence back through its block table reproduces the rows the
    generator drew, bit for bit (decode of a one-hot query would blur this; read the
    pool directly)."""
    w = generate(CONFIGS["decode_b64"])
    dw = DeviceWorkload(w)
    kb = to_bits(dw.k_cache).reshape(-1, w.num_kv_heads, w.head_dim)
    vb = to_bits(dw.v_cache).reshape(-1, w.num_kv_heads, w.head_dim)
    bs = w.block_size
    for s in range(w.num_seqs):
        ctx = int(w.context_lens[s])
        pos = np.arange(ctx)
        rows = w.block_tables[s, pos // bs].astype(np.int64) * bs + pos % bs
        assert np.array_equal(kb[rows], w.logical_k(s))
        assert np.array_equal(vb[rows], w.logical_v(s))


# ------------------------------------------------------------------ decode parity
@pytest.mark.parametrize("name,q_factor", [("tiny_decode", 1.0), ("tiny_decode", 8.0),
                                           ("decode_b64", 1.0), ("decode_b64", 8.0),
                                           ("long_ctx_decode", 1.0), ("long_ctx_decode", 8.0)])
def test_decode_matches_oracle(name, q_factor):
    w = generate(CONFIGS[name], q_factor=q_factor)
    dw = DeviceWorkload(w)
    out = dw.decode()
    assert_close(to_f64(out), oracle_decode(w), f"{name} x{q_factor}")


def test_decode_prefix_sharing_subset_matches_oracle():
    w = generate(CONFIGS["prefix_share_decode"], num_seqs=96)
    dw = DeviceWorkload(w)
    assert_close(to_f64(dw.decode()), oracle_decode(w), "prefix_share 96 seqs")


def test_decode_prefix_sharing_full_size_sampled():
    """All 512 sequences on the GPU in the benchmark's launch configuration; the
    oracle recomputes a sample of sequences one by one."""
    w = generate(CONFIGS["prefix_share_decode"])
    dw = DeviceWorkload(w)
    out = to_f64(dw.decode())
    rng = np.random.default_rng(7)
    seqs = np.sort(rng.choice(w.num_seqs, size=24, replace=False))
    seqs = np.unique(np.concatenate([seqs, [int(np.argmax(w.context_lens)),
                                            int(np.argmin(w.context_lens))]]))
    ref = oracle_decode(w, seqs=seqs)
    assert_close(out[seqs], ref, "prefix_share sampled")


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 64, 256])
def test_decode_shapes_and_ragged_lengths(G, D, bs):
    lens = np.array([1, 2, 63, 64, 65, 255, 256, 257, 700, 1500, 0, 33])
    w = build_workload(kind="decode", context_lens=lens, new_lens=(lens > 0).astype(int),
                       num_q_heads=2 * G, num_kv_heads=2, head_dim=D, block_size=bs,
                       seed=1000 + G * 100 + D + bs)
    dw = DeviceWorkload(w)
    for P in (0, 256):
        out = to_f64(dw.decode(partition_size=P))
        assert_close(out, oracle_decode(w), f"G={G} D={D} bs={bs} P={P}")
        assert np.all(out[lens == 0] == 0.0)


@pytest.mark.parametrize("bs", [16, 256])
def test_decode_sixteen_query_heads_per_kv_head(bs):
    lens = np.array([5, 128, 129, 1000, 3000])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(5, int),
                       num_q_heads=32, num_kv_heads=2, head_dim=128, block_size=bs, seed=40 + bs)
    dw = DeviceWorkload(w)
    for P in (0, 256, 2048):
        assert_close(to_f64(dw.decode(partition_size=P)), oracle_decode(w), f"G=16 bs={bs} P={P}")


def test_single_position_returns_its_value_bit_exact():
    lens = np.array([1, 1, 5, 1])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(4, int), num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=16, seed=77)
    dw = DeviceWorkload(w)
    out = to_bits(dw.decode())
    G = w.num_q_heads // w.num_kv_heads
    for s in np.where(lens == 1)[0]:
        v0 = w.logical_v(int(s))[0]
        for h in range(w.num_q_heads):
            assert np.array_equal(out[s, h], v0[h // G])


# ------------------------------------------------------------------ invariants
def test_split_k_partition_sizes_agree():
    """Split-K merge algebra. Partition sizes that are not multiples of 128 run the
    CUDA-core kernel, whose probabilities stay fp32: splitting changes only the fp32
    summation order, so results stay within one bf16 step of the unsplit ones. The
    tcgen05 kernel (multiples of 128) rounds probabilities to bf16 before P V, so its
    splits agree to that rounding (norm-relative), and every split matches the oracle."""
    w = generate(CONFIGS["long_ctx_decode"])
    dw = DeviceWorkload(w)
    ref = oracle_decode(w)
    base = to_f64(dw.decode(partition_size=32768))       # CUDA-core, one partition
    assert_close(base, ref, "unsplit")
    for P in (320, 576, 1088):                            # CUDA-core, split
        out = to_f64(dw.decode(partition_size=P))
        assert_close(out, ref, f"P={P}")
        assert np.all(np.abs(out - base) <= np.abs(base) * 2.0 ** -7 + 1e-6), P
    tc = {P: to_f64(dw.decode(partition_size=P)) for P in (256, 512, 1024, 2048)}  # tcgen05
    for P, out in tc.items():
        assert_close(out, ref, f"P={P} (tcgen05)")
        assert np.linalg.norm(out - tc[2048]) / np.linalg.norm(tc[2048]) < 5e-3, P


def test_block_permutation_is_bitwise_invariant():
    w = generate(CONFIGS["decode_b64"], num_seqs=16)
    perm = np.random.default_rng(5).permutation(w.num_blocks)
    a = to_bits(DeviceWorkload(w).decode(partition_size=512))
    b = to_bits(DeviceWorkload(relabel_blocks(w, perm)).decode(partition_size=512))
    assert np.array_equal(a, b)


def test_prefix_sharing_is_bitwise_invariant():
    shared = generate(CONFIGS["prefix_share_decode"], num_seqs=64)
    private = generate(CONFIGS["prefix_share_decode"], num_seqs=64, share_prefix=False)
    assert private.num_blocks > shared.num_blocks
    a = to_bits(DeviceWorkload(shared).decode(partition_size=1024))
    b = to_bits(DeviceWorkload(private).decode(partition_size=1024))
    assert np.array_equal(a, b)


def test_decode_is_deterministic():
    w = generate(CONFIGS["decode_b64"])
    dw = DeviceWorkload(w)
    a = to_bits(dw.decode())
    b = to_bits(dw.decode())
    assert np.array_equal(a, b)


def test_bad_block_id_is_reported_not_faulted():
    w = generate(CONFIGS["tiny_decode"])
    dw = DeviceWorkload(w)
    bt = w.block_tables.copy()
    bt[0, 0] = w.num_blocks + 100
    pa.pa_set_debug_checks(True)
    try:
        out = torch.empty_like(dw.q)
        ws, P = pa.decode_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                    w.max_context_len, 256)
        with pytest.raises(pa.PAError) as e:
            pa.pa_decode(out, dw.q, dw.k_cache, dw.v_cache, i32_dev(bt), dw.context_lens, w.scale,
                         w.max_context_len, P, ws)
        assert e.value.status == 3
    finally:
        pa.pa_set_debug_checks(True)
    # the context stays usable
    assert_close(to_f64(dw.decode()), oracle_decode(w), "after bad index")


@pytest.mark.parametrize("P", [0, 128])
def test_decode_many_one_tile_items(P):
    """640 sequences of at most 130 positions over 8 kv heads: thousands of work items of
    one or two tiles, so the tensor-core issuer crosses an item boundary at almost every
    tile (its score cursor runs ahead across items) and each CTA runs dozens of items,
    reusing every item slot, S buffer, P buffer and O accumulator many times."""
    rng = np.random.default_rng(64)
    lens = rng.integers(1, 131, size=640)
    lens[:6] = [1, 2, 127, 128, 129, 130]
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones_like(lens),
                       num_q_heads=16, num_kv_heads=8, head_dim=128, block_size=16,
                       seed=6400 + P)
    dw = DeviceWorkload(w)
    got = to_f64(dw.decode(P))
    assert_close(got, oracle_decode(w), f"one-tile items P={P}")
    # and the same bits when the batch is decoded again (every item slot reused)
    again = to_f64(dw.decode(P))
    assert np.array_equal(got, again)
