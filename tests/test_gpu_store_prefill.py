"""pa_store_prefill: the new tokens' K/V rows stored and the causal prefill run in one
launch. Its output must equal pa_store_kvcache followed by pa_prefill bit for bit (the
attention reads the same bits, from k / v instead of the pool), and the pools after the
call must equal the oracle's store byte for byte."""
import numpy as np
import pytest
import torch

import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import (DeviceWorkload, assert_close, i32_dev, oracle_pools,
                               oracle_prefill, to_bits, to_f64)
from workloads import CONFIGS, build_workload, generate

pytestmark = pytest.mark.gpu


def fused(w, slots=None):
    dw = DeviceWorkload(w, store_new=False)
    out = torch.empty_like(dw.q)
    max_q = int(np.max(np.diff(w.cu_seqlens_q))) if w.num_seqs else 0
    pa.pa_store_prefill(dw.new_k, dw.new_v, dw.new_slots if slots is None else slots, out, dw.q,
                        dw.k_cache, dw.v_cache, dw.block_tables, dw.cu_seqlens_q, dw.context_lens,
                        w.scale, max_q)
    return out, dw


def check_equal_to_store_then_prefill(w, what):
    got, dw = fused(w)
    want = DeviceWorkload(w).prefill()
    assert np.array_equal(to_bits(got), to_bits(want)), f"{what}: differs from store + prefill"
    kc, vc = oracle_pools(w)
    assert np.array_equal(to_bits(dw.k_cache), kc), f"{what}: K pool"
    assert np.array_equal(to_bits(dw.v_cache), vc), f"{what}: V pool"
    return got


@pytest.mark.parametrize("bs", [16, 64, 256])
@pytest.mark.parametrize("G", [1, 2, 4])
def test_store_prefill_ragged_shapes(bs, G):
    """First new positions aligned and not aligned to a 128-position tile (the tile
    that holds both cached and new rows is patched from k / v), whole sequences new,
    one new token, odd counts of query tiles."""
    ctx = np.array([300, 129, 1000, 130, 128, 1, 640, 77, 390])
    new = np.array([300, 1, 200, 3, 128, 1, 129, 77, 262])
    w = build_workload(kind="prefill", context_lens=ctx, new_lens=new, num_q_heads=2 * G,
                       num_kv_heads=2, head_dim=128, block_size=bs, seed=600 + bs + G)
    got = check_equal_to_store_then_prefill(w, f"bs={bs} G={G}")
    assert_close(to_f64(got), oracle_prefill(w), f"bs={bs} G={G} vs oracle")


def test_store_prefill_chunked_full_size():
    """The full 32 x (2048 + 512) chunked prefill step in one launch."""
    w = generate(CONFIGS["chunked_prefill"])
    check_equal_to_store_then_prefill(w, "chunked_prefill")


def test_store_prefill_subset_matches_oracle():
    w = generate(CONFIGS["chunked_prefill"], num_seqs=3)
    got = check_equal_to_store_then_prefill(w, "chunked_prefill 3 seqs")
    assert_close(to_f64(got), oracle_prefill(w), "chunked_prefill 3 seqs vs oracle")


def test_store_prefill_reports_a_slot_off_its_position():
    """A slot that is not the block table's slot for the token's position is not
    written and is reported; the other rows are stored, and the attention (which reads
    the new rows from k / v) is unchanged."""
    ctx = np.array([400, 200])
    new = np.array([150, 200])
    w = build_workload(kind="prefill", context_lens=ctx, new_lens=new, num_q_heads=4,
                       num_kv_heads=2, head_dim=128, block_size=64, seed=611)
    slots = w.new_slots.copy()
    spare = int(np.setdiff1d(np.arange(w.num_blocks * w.block_size), slots)[0])
    bad = 7
    slots[bad] = spare
    pa.pa_set_debug_checks(True)
    with pytest.raises(pa.PAError) as e:
        fused(w, i32_dev(slots))
    assert e.value.status == 3
    got, dw = fused(w, i32_dev(np.where(np.arange(len(slots)) == bad, -1, slots).astype(np.int32)))
    ref = w.new_slots.copy()
    ref[bad] = -1
    kc, vc = w.empty_pool(), w.empty_pool()
    import oracle
    kc, vc = oracle.store_kvcache(kc, vc, w.setup_k, w.setup_v, w.setup_slots)
    kc, vc = oracle.store_kvcache(kc, vc, w.new_k, w.new_v, ref)
    assert np.array_equal(to_bits(dw.k_cache), kc)
    assert np.array_equal(to_bits(dw.v_cache), vc)
    assert_close(to_f64(got), oracle_prefill(w), "attention from the new rows")
