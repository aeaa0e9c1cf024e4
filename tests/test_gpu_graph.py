"""Decode captured into a CUDA graph. The capture fixes the call's counter tag, so the
graph clears the workspace's counter block before the call (include/pa.h); every
replay must then equal the eager call bit for bit, for pa_decode with split contexts
and for the one-launch store + decode step."""
import numpy as np
import pytest
import torch

import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import DeviceWorkload, i32_dev
from workloads import CONFIGS, generate

pytestmark = pytest.mark.gpu


def counter_elems(w):
    return -(-(8 * (1 + w.num_seqs * w.num_q_heads)) // 256) * 256 // 4


def capture(fn, ws, n):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        ws[:n].zero_()
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ws[:n].zero_()
        fn()
    return g


@pytest.mark.parametrize("fused", [False, True])
def test_graph_replays_equal_the_eager_call(fused):
    w = generate(CONFIGS["decode_b64"], num_seqs=24)
    dw = DeviceWorkload(w, store_new=not fused)
    ws, P = pa.decode_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                w.max_context_len, 256)
    out_e = torch.empty_like(dw.q)
    out_g = torch.empty_like(dw.q)

    def call(out):
        if fused:
            pa.pa_store_decode(dw.new_k, dw.new_v, dw.new_slots, out, dw.q, dw.k_cache,
                               dw.v_cache, dw.block_tables, dw.context_lens, w.scale,
                               w.max_context_len, P, ws)
        else:
            pa.pa_decode(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens,
                         w.scale, w.max_context_len, P, ws)

    call(out_e)
    torch.cuda.synchronize()
    pa.pa_set_debug_checks(False)      # a synchronising check cannot run inside a capture
    try:
        g = capture(lambda: call(out_g), ws, counter_elems(w))
        for _ in range(3):
            out_g.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(out_g.view(torch.int16), out_e.view(torch.int16))
        del g
    finally:
        pa.pa_set_debug_checks(True)
    assert pa.pa_check_device_errors() == 0
