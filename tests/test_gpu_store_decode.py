"""pa_store_decode: one call that stores each sequence's new K/V row and decodes.

Its result and the pool it leaves must equal pa_store_kvcache followed by pa_decode
(bit for bit: the same rows are read in the same order), and both must match the
oracle. The tensor-core path stores inside the decode kernel; head dim 64 and
partition sizes that kernel does not take run a checked store kernel first.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import (DeviceWorkload, assert_close, bf16_dev, i32_dev, oracle_decode,
                               oracle_pools, to_bits, to_f64)
from workloads import CONFIGS, build_workload, generate

pytestmark = pytest.mark.gpu


def per_seq_rows(w):
    """New rows and slots indexed by sequence ([B, Hkv, D] bits, [B] int32, -1 = none)."""
    B = w.num_seqs
    k = np.zeros((B, w.num_kv_heads, w.head_dim), dtype=np.uint16)
    v = np.zeros_like(k)
    slots = np.full(B, -1, dtype=np.int32)
    seqs = np.nonzero(w.new_lens)[0]
    assert np.all(w.new_lens[seqs] == 1) and len(seqs) == len(w.new_slots)
    k[seqs], v[seqs], slots[seqs] = w.new_k, w.new_v, w.new_slots
    # the slot of each stored row is the sequence's last position, as the block table maps it
    bs = w.block_size
    last = w.context_lens[seqs] - 1
    assert np.array_equal(slots[seqs], w.block_tables[seqs, last // bs] * bs + last % bs)
    return k, v, slots


def fused(dw, k, v, slots, partition_size=0):
    w = dw.w
    out = torch.empty_like(dw.q)
    ws, P = pa.decode_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                w.max_context_len, partition_size)
    pa.pa_store_decode(bf16_dev(k), bf16_dev(v), i32_dev(slots), out, dw.q, dw.k_cache, dw.v_cache,
                       dw.block_tables, dw.context_lens, w.scale, w.max_context_len, P, ws)
    return out


@pytest.mark.parametrize("name,P", [("tiny_decode", 0), ("decode_b64", 0), ("decode_b64", 256),
                                    ("decode_b64", 2048), ("decode_b64", 320),
                                    ("long_ctx_decode", 0)])
def test_store_decode_equals_store_then_decode(name, P):
    w = generate(CONFIGS[name])
    k, v, slots = per_seq_rows(w)
    one = DeviceWorkload(w, store_new=False)
    out = fused(one, k, v, slots, P)
    two = DeviceWorkload(w)                     # pa_store_kvcache, then pa_decode
    ref = two.decode(partition_size=P)
    assert np.array_equal(to_bits(out), to_bits(ref)), name
    kc, vc = oracle_pools(w)
    assert np.array_equal(to_bits(one.k_cache), kc)
    assert np.array_equal(to_bits(one.v_cache), vc)
    assert_close(to_f64(out), oracle_decode(w), f"store_decode {name} P={P}")


@pytest.mark.parametrize("G,bs", [(1, 16), (4, 64), (8, 256), (16, 16)])
def test_store_decode_shapes_and_empty_contexts(G, bs):
    lens = np.array([1, 2, 127, 128, 129, 700, 0, 1500, 33])
    w = build_workload(kind="decode", context_lens=lens, new_lens=(lens > 0).astype(int),
                       num_q_heads=2 * G, num_kv_heads=2, head_dim=128, block_size=bs,
                       seed=3000 + G * 10 + bs)
    k, v, slots = per_seq_rows(w)
    for P in (0, 256):
        one = DeviceWorkload(w, store_new=False)
        out = to_f64(fused(one, k, v, slots, P))
        assert_close(out, oracle_decode(w), f"G={G} bs={bs} P={P}")
        assert np.all(out[lens == 0] == 0.0)
        kc, vc = oracle_pools(w)
        assert np.array_equal(to_bits(one.k_cache), kc)
        assert np.array_equal(to_bits(one.v_cache), vc)


def test_store_decode_skips_minus_one():
    w = generate(CONFIGS["decode_b64"], num_seqs=16)
    k, v, slots = per_seq_rows(w)
    skip = slots.copy()
    skip[::3] = -1
    one = DeviceWorkload(w, store_new=False)
    before = to_bits(one.k_cache).reshape(-1, w.num_kv_heads, w.head_dim).copy()
    out = fused(one, k, v, skip)
    two = DeviceWorkload(w, store_new=False)
    pa.pa_store_kvcache(bf16_dev(k), bf16_dev(v), two.k_cache, two.v_cache, i32_dev(skip))
    assert np.array_equal(to_bits(out), to_bits(two.decode()))
    after = to_bits(one.k_cache).reshape(-1, w.num_kv_heads, w.head_dim)
    for s in range(0, 16, 3):
        assert np.array_equal(after[slots[s]], before[slots[s]])      # left as it was
    for s in range(1, 16, 3):
        assert np.array_equal(after[slots[s]], k[s])


@pytest.mark.parametrize("name", ["decode_b64", "tiny_decode"])
def test_store_decode_rejects_a_slot_that_is_not_the_last_position(name):
    """A slot elsewhere in the context could be read before it is written: it is
    reported (PA_ERR_BAD_INDEX) and not stored, and the context stays usable."""
    w = generate(CONFIGS[name])
    k, v, slots = per_seq_rows(w)
    s = int(np.argmax(w.context_lens))
    pos = int(w.context_lens[s]) - 2
    wrong = slots.copy()
    wrong[s] = int(w.block_tables[s, pos // w.block_size]) * w.block_size + pos % w.block_size
    one = DeviceWorkload(w, store_new=False)
    before = to_bits(one.k_cache).reshape(-1, w.num_kv_heads, w.head_dim).copy()
    pa.pa_set_debug_checks(True)
    with pytest.raises(pa.PAError) as e:
        fused(one, k, v, wrong)
    assert e.value.status == 3
    assert pa.pa_check_device_errors() == 0
    after = to_bits(one.k_cache).reshape(-1, w.num_kv_heads, w.head_dim)
    assert np.array_equal(after[wrong[s]], before[wrong[s]])
    assert np.array_equal(after[slots[s]], before[slots[s]])
    # a correct call afterwards works
    out = fused(one, k, v, slots)
    assert_close(to_f64(out), oracle_decode(w), f"{name} after a rejected slot")
