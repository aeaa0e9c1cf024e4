"""Copy-on-write of shared blocks on the GPU (pa_copy_blocks), bit-exact against the
oracle's copy, and a decode step that appends into private copies of shared blocks."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import DeviceWorkload, assert_close, i32_dev, to_bits, to_f64
from tests.test_gpu_store_decode import fused, per_seq_rows
from workloads import CONFIGS, copy_on_write_append, generate

pytestmark = pytest.mark.gpu


def random_pools(nb, bs, hkv, d, seed):
    rng = np.random.default_rng(seed)
    k = rng.integers(0, 1 << 16, size=(nb, bs, hkv, d), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(nb, bs, hkv, d), dtype=np.uint16)
    return k, v


def dev(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("bs,hkv,d", [(64, 8, 128), (16, 2, 64), (256, 8, 128), (16, 1, 64)])
def test_copy_blocks_bit_exact(bs, hkv, d):
    nb = 40
    k, v = random_pools(nb, bs, hkv, d, seed=bs + hkv + d)
    rng = np.random.default_rng(9)
    ids = rng.permutation(nb)
    src, dst = ids[:12].astype(np.int32), ids[12:24].astype(np.int32)
    kd, vd = dev(k), dev(v)
    pa.pa_copy_blocks(kd, vd, i32_dev(src), i32_dev(dst))
    ok, ov = oracle.copy_blocks(k, v, src, dst)
    assert np.array_equal(to_bits(kd), ok)
    assert np.array_equal(to_bits(vd), ov)


def test_copy_blocks_many_pairs_and_noops():
    nb = 300
    k, v = random_pools(nb, 16, 2, 64, seed=5)
    src = np.arange(0, 150, dtype=np.int32)
    dst = np.arange(150, 300, dtype=np.int32)
    src[7] = dst[7]                # src == dst: nothing moves
    kd, vd = dev(k), dev(v)
    pa.pa_copy_blocks(kd, vd, i32_dev(src), i32_dev(dst))
    keep = np.ones(150, bool)
    keep[7] = False
    ok, ov = oracle.copy_blocks(k, v, src[keep], dst[keep])
    assert np.array_equal(to_bits(kd), ok)
    assert np.array_equal(to_bits(vd), ov)


def test_copy_blocks_reports_bad_ids():
    k, v = random_pools(8, 16, 2, 64, seed=6)
    kd, vd = dev(k), dev(v)
    pa.pa_set_debug_checks(True)
    with pytest.raises(pa.PAError) as e:
        pa.pa_copy_blocks(kd, vd, i32_dev(np.array([1, 2], np.int32)), i32_dev(np.array([8, 3], np.int32)))
    assert e.value.status == 3
    assert pa.pa_check_device_errors() == 0
    # the good pair was copied, the bad one skipped
    ok, ov = oracle.copy_blocks(k, v, np.array([2]), np.array([3]))
    assert np.array_equal(to_bits(kd), ok)
    assert np.array_equal(to_bits(vd), ov)


@pytest.mark.parametrize("num_seqs", [96, None])
def test_copy_on_write_then_append_decode(num_seqs):
    """Prefix-sharing batch: copy the shared blocks the sequences are about to append
    into, then one pa_store_decode; output and pools match the oracle's pipeline."""
    w = generate(CONFIGS["prefix_share_decode"], num_seqs=num_seqs)
    w2, src, dst = copy_on_write_append(w)
    assert len(src) > 0
    dw = DeviceWorkload(w2, store_new=False)       # the pools as the sequences left them
    pa.pa_copy_blocks(dw.k_cache, dw.v_cache, i32_dev(src), i32_dev(dst))
    k, v, slots = per_seq_rows(w2)
    out = to_f64(fused(dw, k, v, slots))
    kc, vc = w2.empty_pool(), w2.empty_pool()
    kc, vc = oracle.store_kvcache(kc, vc, w2.setup_k, w2.setup_v, w2.setup_slots)
    kc, vc = oracle.copy_blocks(kc, vc, src, dst)
    kc, vc = oracle.store_kvcache(kc, vc, w2.new_k, w2.new_v, w2.new_slots)
    assert np.array_equal(to_bits(dw.k_cache), kc)
    assert np.array_equal(to_bits(dw.v_cache), vc)
    if num_seqs is not None:
        ref = oracle.decode(w2.q, kc, vc, w2.block_tables, w2.context_lens, w2.scale)
        assert_close(out, ref, "cow append")
    else:
        seqs = np.unique(np.concatenate([np.arange(0, w2.num_seqs, 37),
                                         [int(np.argmax(w2.context_lens))]]))
        ref = oracle.decode(w2.q[seqs], kc, vc, w2.block_tables[seqs], w2.context_lens[seqs], w2.scale)
        assert_close(out[seqs], ref, "cow append sampled")
