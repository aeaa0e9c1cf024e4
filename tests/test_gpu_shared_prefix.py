"""pa_decode_shared_prefix: decode of a batch whose sequences share their first blocks
(one common prompt), with the shared prefix attended once for all sequences.

Checked against the fp64 oracle within the decode bar (ragged shapes, the prefix-sharing
configuration on a 96-sequence subset and at full size on sampled sequences), for
bitwise invariance under relabelling the physical blocks, and for the report of a block
table that does not hold the shared blocks."""
import numpy as np
import pytest
import torch

import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import (DeviceWorkload, assert_close, i32_dev, oracle_decode, to_bits,
                               to_f64)
from workloads import CONFIGS, build_workload, generate, relabel_blocks

pytestmark = pytest.mark.gpu


def shared_blocks_of(w, shared_len):
    """The prefix's physical blocks: those of the longest sequence (every sequence holds
    them at the prefix positions it uses)."""
    s = int(np.argmax(w.context_lens))
    nb = shared_len // w.block_size
    assert int(w.context_lens[s]) >= shared_len
    return w.block_tables[s, :nb].astype(np.int32)


def shared_decode(dw, shared_len, partition_size=0, blocks=None, bt=None):
    w = dw.w
    out = torch.empty_like(dw.q)
    ws, P = pa.shared_prefix_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                       w.max_context_len, shared_len, partition_size)
    sb = i32_dev(shared_blocks_of(w, shared_len) if blocks is None else blocks)
    pa.pa_decode_shared_prefix(out, dw.q, dw.k_cache, dw.v_cache,
                               dw.block_tables if bt is None else bt, dw.context_lens, w.scale,
                               w.max_context_len, sb, shared_len, P, ws)
    return out


@pytest.mark.parametrize("G", [1, 4, 16])
@pytest.mark.parametrize("bs", [16, 64, 256])
def test_shared_prefix_ragged(G, bs):
    """Contexts shorter than, equal to and longer than the prefix, empty and one-long,
    split and unsplit suffixes."""
    S = 256
    lens = np.array([0, 1, 100, 255, 256, 257, 300, 1000, 2100, 128, 40, 700])
    w = build_workload(kind="decode", context_lens=lens, new_lens=(lens > 0).astype(int),
                       num_q_heads=2 * G, num_kv_heads=2, head_dim=128, block_size=bs,
                       seed=700 + G + bs, shared_prefix_len=S)
    dw = DeviceWorkload(w)
    ref = oracle_decode(w)
    for P in (0, 128, 512):
        got = to_f64(shared_decode(dw, S, P))
        assert_close(got, ref, f"G={G} bs={bs} P={P}")
        assert np.all(got[lens == 0] == 0)


def test_shared_prefix_subset_matches_oracle():
    w = generate(CONFIGS["prefix_share_decode"], num_seqs=96)
    dw = DeviceWorkload(w)
    got = to_f64(shared_decode(dw, 1024))
    assert_close(got, oracle_decode(w), "prefix_share 96 seqs (shared prefix)")
    plain = to_f64(dw.decode())
    assert np.linalg.norm(got - plain) / np.linalg.norm(plain) < 5e-3


def test_shared_prefix_full_size_sampled():
    """All 512 sequences in the benchmark's launch configuration; the oracle recomputes a
    sample, including the longest and the shortest sequence."""
    w = generate(CONFIGS["prefix_share_decode"])
    dw = DeviceWorkload(w)
    out = to_f64(shared_decode(dw, 1024))
    rng = np.random.default_rng(8)
    seqs = np.sort(rng.choice(w.num_seqs, size=24, replace=False))
    seqs = np.unique(np.concatenate([seqs, [int(np.argmax(w.context_lens)),
                                            int(np.argmin(w.context_lens))]]))
    assert_close(out[seqs], oracle_decode(w, seqs=seqs), "prefix_share sampled (shared prefix)")


def test_shared_prefix_block_permutation_is_bitwise_invariant():
    w = generate(CONFIGS["prefix_share_decode"], num_seqs=64)
    perm = np.random.default_rng(9).permutation(w.num_blocks)
    w2 = relabel_blocks(w, perm)
    a = to_bits(shared_decode(DeviceWorkload(w), 1024, 512))
    b = to_bits(shared_decode(DeviceWorkload(w2), 1024, 512))
    assert np.array_equal(a, b)


def test_shared_prefix_reports_a_table_without_the_shared_blocks():
    w = generate(CONFIGS["prefix_share_decode"], num_seqs=32)
    dw = DeviceWorkload(w)
    s = int(np.argmax(w.context_lens))
    bt = w.block_tables.copy()
    other = int(np.setdiff1d(np.arange(w.num_blocks), bt[s, :16])[0])
    bt[s, 3] = other
    pa.pa_set_debug_checks(True)
    with pytest.raises(pa.PAError) as e:
        shared_decode(dw, 1024, blocks=shared_blocks_of(w, 1024), bt=i32_dev(bt))
    assert e.value.status == 3


def test_shared_prefix_two_units_per_cta():
    """A batch large enough that the prefix pass runs two 128-row units per CTA (with 16
    query heads per kv head a unit holds 8 sequences; 320 sequences x 8 kv heads fill
    more than one unit per SM), checked against the oracle on sampled sequences,
    contexts shorter than, equal to and just past the prefix among them."""
    S = 128
    rng = np.random.default_rng(21)
    lens = rng.integers(1, 420, size=320)
    lens[:4] = [1, 127, 128, 129]
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones_like(lens),
                       num_q_heads=128, num_kv_heads=8, head_dim=128, block_size=64,
                       seed=2100, shared_prefix_len=S)
    dw = DeviceWorkload(w)
    out = to_f64(shared_decode(dw, S))
    seqs = np.unique(np.concatenate([np.arange(6), rng.choice(w.num_seqs, size=18, replace=False),
                                     [w.num_seqs - 1]]))
    assert_close(out[seqs], oracle_decode(w, seqs=seqs), "two units per CTA (sampled)")
