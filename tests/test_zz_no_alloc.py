"""pa_decode_no_alloc: decode for callers that cannot allocate device memory.

Such callers (a runtime that fixes all of its GPU memory at start-up, or a host
program that only binds the C ABI and has no CUDA allocator) cannot hand pa_decode
a workspace; this entry point uses the library's own fixed scratch array instead.
The test drives it through the C ABI and checks it on two calls in a row with
different workloads, so the second call runs on whatever the first left in the
shared array: bit for bit against pa_decode (which gets a caller-allocated
workspace) at the same partition size, and against the oracle within the bar.

Kept in its own file, named to be collected after every other test.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import DeviceWorkload, assert_close, oracle_decode, to_bits
from workloads import CONFIGS, generate

pytestmark = pytest.mark.gpu


def _no_alloc(dw):
    w = dw.w
    out = torch.empty_like(dw.q)
    pa.pa_decode_no_alloc(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens,
                          w.scale, w.max_context_len)
    return out


def test_no_alloc_decode_matches_workspace_decode_on_two_calls():
    """Two calls in a row (the second runs on whatever the first left in the shared
    array): each equals pa_decode at the same partition size bit for bit, and matches
    the oracle within the decode bar."""
    first = DeviceWorkload(generate(CONFIGS["decode_b64"]))
    second = DeviceWorkload(generate(CONFIGS["long_ctx_decode"]))
    for dw in (first, second):
        w = dw.w
        P = pa.pa_decode_default_partition(w.num_seqs, w.num_kv_heads, w.max_context_len)
        need = pa.pa_decode_workspace_size(w.num_seqs, w.num_q_heads, w.head_dim,
                                           w.max_context_len, P)
        assert 0 < need <= pa.DECODE_NO_ALLOC_SCRATCH_BYTES  # both calls really use the scratch
        assert P < w.max_context_len                         # and both split their contexts
    ref1, ref2 = to_bits(first.decode()), to_bits(second.decode())
    got1 = to_bits(_no_alloc(first))
    got2 = to_bits(_no_alloc(second))
    torch.cuda.synchronize()
    assert np.array_equal(got1, ref1), "no-alloc call 1 differs from pa_decode"
    assert np.array_equal(got2, ref2), "no-alloc call 2 differs from pa_decode"
    assert_close(bits_to_f64(got1), oracle_decode(first.w), "no-alloc call 1 vs oracle")
    assert_close(bits_to_f64(got2), oracle_decode(second.w), "no-alloc call 2 vs oracle")


def bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_no_alloc_rejects_sizes_beyond_its_scratch():
    w = generate(CONFIGS["decode_b64"], num_seqs=8)
    dw = DeviceWorkload(w)
    # 8 sequences x 16 heads x (4096 / 64) partitions x 130 floats = 4.3 MB fits;
    # ask for a context bound that needs more than the fixed array holds
    P = 64
    max_ctx = w.max_blocks_per_seq * w.block_size
    need = pa.pa_decode_workspace_size(w.num_seqs, w.num_q_heads, w.head_dim, max_ctx, P)
    if need <= pa.DECODE_NO_ALLOC_SCRATCH_BYTES:
        bt = torch.full((w.num_seqs, 256), -1, dtype=torch.int32, device="cuda")
        bt[:, :w.max_blocks_per_seq] = dw.block_tables
        max_ctx = 256 * w.block_size
        need = pa.pa_decode_workspace_size(w.num_seqs, w.num_q_heads, w.head_dim, max_ctx, P)
    else:
        bt = dw.block_tables
    assert need > pa.DECODE_NO_ALLOC_SCRATCH_BYTES
    out = torch.empty_like(dw.q)
    with pytest.raises(pa.PAError, match="more than the library's fixed") as e:
        pa.pa_decode_no_alloc(out, dw.q, dw.k_cache, dw.v_cache, bt, dw.context_lens, w.scale,
                              max_ctx, P)
    assert e.value.status == 2
