"""A bounded device wait that runs out is reported, and leaves the GPU usable.

The tensor-core kernels' roles wait for one another on shared-memory barriers, each
wait bounded in time. pa_set_wait_limit_ns shortens that bound for later calls (the
waits a CTA makes before it exits, for its own copies and tensor-core operations,
keep the full limit). With a bound of 1 ns, a wait for a tile still in flight runs out
at once: the kernel records PA_ERR_TIMEOUT, every role winds down, and the call returns
that status (debug checks read the error word). The next call, with the default bound,
must be a normal one: within the parity bar against the oracle.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_442_b200 as pa
from tests.gpu_helpers import DeviceWorkload, assert_close, oracle_decode, oracle_prefill, to_f64
from workloads import build_workload

pytestmark = pytest.mark.gpu


def _run_timed_out(fn):
    pa.pa_set_debug_checks(True)
    pa.pa_set_wait_limit_ns(1)
    try:
        with pytest.raises(pa.PAError) as e:
            fn()
        assert e.value.status == 5, e.value
    finally:
        pa.pa_set_wait_limit_ns(0)
    torch.cuda.synchronize()
    assert pa.pa_check_device_errors() == 0   # the word was read and cleared by the call


def test_decode_wait_that_runs_out_is_reported():
    lens = np.array([700, 129, 3000, 1, 2048])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(5, int), num_q_heads=16,
                       num_kv_heads=8, head_dim=128, block_size=64, seed=31)
    dw = DeviceWorkload(w)
    _run_timed_out(lambda: dw.decode(partition_size=256))
    assert_close(to_f64(dw.decode(partition_size=256)), oracle_decode(w), "decode after a timeout")


def test_prefill_wait_that_runs_out_is_reported():
    w = build_workload(kind="prefill", context_lens=np.array([700, 300]),
                       new_lens=np.array([200, 300]), num_q_heads=8, num_kv_heads=2, head_dim=128,
                       block_size=64, seed=32)
    dw = DeviceWorkload(w)
    _run_timed_out(dw.prefill)
    assert_close(to_f64(dw.prefill()), oracle_prefill(w), "prefill after a timeout")


def test_fp8_decode_wait_that_runs_out_is_reported():
    from tests.test_gpu_fp8 import Fp8Pools, gpu_decode_fp8, oracle_decode_fp8
    lens = np.array([700, 129, 3000, 1])
    w = build_workload(kind="decode", context_lens=lens, new_lens=np.ones(4, int), num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=64, seed=33)
    pools = Fp8Pools(w)
    _run_timed_out(lambda: gpu_decode_fp8(w, pools, 256))
    assert_close(gpu_decode_fp8(w, pools, 256), oracle_decode_fp8(w, pools.host),
                 "fp8 decode after a timeout")
