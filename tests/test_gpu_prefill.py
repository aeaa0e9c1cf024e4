"""GPU parity of the tcgen05 causal paged prefill against the CPU oracle."""
import numpy as np
import pytest

from tests.gpu_helpers import (DeviceWorkload, assert_close, oracle_decode, oracle_pools,
                               oracle_prefill, to_bits, to_f64)
from workloads import CONFIGS, build_workload, generate, relabel_blocks

import oracle

pytestmark = pytest.mark.gpu


def test_prefill_subset_matches_oracle():
    w = generate(CONFIGS["chunked_prefill"], num_seqs=3)
    dw = DeviceWorkload(w)
    assert_close(to_f64(dw.prefill()), oracle_prefill(w), "chunked_prefill 3 seqs")


def test_prefill_peaked_subset_matches_oracle():
    w = generate(CONFIGS["chunked_prefill"], num_seqs=2, q_factor=8.0)
    dw = DeviceWorkload(w)
    assert_close(to_f64(dw.prefill()), oracle_prefill(w), "chunked_prefill peaked")


def test_prefill_full_size_sampled():
    """The full 32 x (2048 + 512) workload on the GPU; the oracle recomputes a sample
    of (sequence, query head) pairs one at a time."""
    w = generate(CONFIGS["chunked_prefill"])
    dw = DeviceWorkload(w)
    out = to_f64(dw.prefill())
    kc, vc = oracle_pools(w)
    rng = np.random.default_rng(3)
    for s in rng.choice(w.num_seqs, size=3, replace=False):
        s = int(s)
        q0, q1 = int(w.cu_seqlens_q[s]), int(w.cu_seqlens_q[s + 1])
        cu = np.array([0, q1 - q0], np.int32)
        heads = rng.choice(w.num_q_heads, size=4, replace=False)
        ref = oracle.prefill(w.q[q0:q1], kc, vc, w.block_tables[s:s + 1], cu,
                             w.context_lens[s:s + 1], w.scale)
        assert_close(out[q0:q1][:, heads], ref[:, heads], f"seq {s} heads {heads}")


@pytest.mark.parametrize("bs", [16, 64, 256])
@pytest.mark.parametrize("G", [1, 2, 4])
def test_prefill_ragged_shapes(bs, G):
    ctx = np.array([300, 129, 1000, 130, 128, 1, 640, 77])
    new = np.array([300, 1, 200, 3, 128, 1, 129, 77])
    w = build_workload(kind="prefill", context_lens=ctx, new_lens=new, num_q_heads=2 * G,
                       num_kv_heads=2, head_dim=128, block_size=bs, seed=500 + bs + G)
    dw = DeviceWorkload(w)
    assert_close(to_f64(dw.prefill()), oracle_prefill(w), f"bs={bs} G={G}")


def test_prefill_one_token_equals_decode():
    lens = np.array([700, 1, 129, 2048, 300])
    wd = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(5, int),
                        num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=256, seed=91)
    dw = DeviceWorkload(wd)
    dec = to_f64(dw.decode())
    wp = build_workload(kind="prefill", context_lens=lens, new_lens=np.ones(5, int),
                        num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=256, seed=91)
    assert np.array_equal(wp.q, wd.q)
    pre = to_f64(DeviceWorkload(wp).prefill())
    ref = oracle_decode(wd)
    assert_close(dec, ref, "decode")
    assert_close(pre, ref, "prefill of one token")


def test_prefill_is_deterministic():
    w = generate(CONFIGS["chunked_prefill"], num_seqs=4)
    dw = DeviceWorkload(w)
    assert np.array_equal(to_bits(dw.prefill()), to_bits(dw.prefill()))


@pytest.mark.parametrize("bs", [64, 256])
def test_prefill_block_permutation_is_bitwise_invariant(bs):
    """Relabelling the physical blocks (data and tables moved together) gives the same
    bits: the kernel's arithmetic depends only on logical positions."""
    ctx = np.array([700, 300, 1000, 129])
    new = np.array([200, 300, 129, 1])
    w = build_workload(kind="prefill", context_lens=ctx, new_lens=new, num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=bs, seed=900 + bs)
    perm = np.random.default_rng(bs).permutation(w.num_blocks)
    a = to_bits(DeviceWorkload(w).prefill())
    b = to_bits(DeviceWorkload(relabel_blocks(w, perm)).prefill())
    assert np.array_equal(a, b)
