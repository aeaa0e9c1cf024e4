"""The C ABI library loads, exports every function include/pa.h declares, and its
host-side validation rejects bad arguments before any launch (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import paged_kv_cache_442_b200 as pa
from paged_kv_cache_442_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return pa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(pa.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (pa_\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_host_only_calls(lib):
    assert pa.pa_version() == 100
    assert pa.pa_status_string(0) == "PA_OK"
    assert pa.pa_status_string(5) == "PA_ERR_TIMEOUT"
    # workspace: 256-aligned counters (1 + B*Hq of 8 bytes), then [B, Hq, parts, D + 2]
    # fp32 partials when the context is split
    counters = -(-(8 * (1 + 8 * 32)) // 256) * 256
    assert pa.pa_decode_workspace_size(8, 32, 128, 32768, 1024) == counters + 8 * 32 * 32 * 130 * 4
    assert pa.pa_decode_workspace_size(8, 32, 128, 1024, 1024) == counters
    assert pa.pa_decode_workspace_size(0, 32, 128, 1024, 256) == 0


def desc(nb=16, bs=16, hkv=2, d=128):
    return pa.pa_cache_desc(nb, bs, hkv, d)


NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first


@pytest.mark.parametrize("bad", [desc(bs=12), desc(bs=8), desc(bs=2048), desc(d=96), desc(nb=0),
                                 desc(hkv=0), desc(nb=1 << 22, bs=1024)])
def test_bad_cache_shapes_are_rejected(lib, bad):
    st = lib.pa_store_kvcache(FAKE, FAKE, FAKE, FAKE, bad, FAKE, 4, NULL)
    assert st == 1
    st = lib.pa_decode(FAKE, FAKE, FAKE, FAKE, bad, FAKE, 4, FAKE, 2, 4, 0.1, 32, 0, NULL, 0, NULL)
    assert st == 1


def test_store_argument_checks(lib):
    assert lib.pa_store_kvcache(NULL, FAKE, FAKE, FAKE, desc(), FAKE, 4, NULL) == 1
    assert lib.pa_store_kvcache(FAKE, FAKE, FAKE, FAKE, desc(), FAKE, -1, NULL) == 1
    misaligned = ctypes.c_void_p((1 << 20) + 8)
    assert lib.pa_store_kvcache(misaligned, FAKE, FAKE, FAKE, desc(), FAKE, 4, NULL) == 1
    assert lib.pa_store_kvcache(NULL, NULL, NULL, NULL, desc(), NULL, 0, NULL) == 0  # no-op


def test_decode_argument_checks(lib):
    d = desc(hkv=2)
    # Hq not a multiple of Hkv
    assert lib.pa_decode(FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 3, 0.1, 32, 0, NULL, 0, NULL) == 1
    # group of 3 query heads per kv head: valid but not implemented
    assert lib.pa_decode(FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 6, 0.1, 32, 0, NULL, 0, NULL) == 2
    # context longer than the block table can address
    assert lib.pa_decode(FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 4, 0.1, 65, 0, NULL, 0, NULL) == 1
    # non-finite scale
    assert lib.pa_decode(FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 4, float("nan"), 32, 0, NULL, 0,
                         NULL) == 1
    # partition size not a multiple of 64
    assert lib.pa_decode(FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 4, 0.1, 32, 100, NULL, 0, NULL) == 1
    # split needs a workspace
    assert lib.pa_decode(FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 4, 0.1, 64, 64, NULL, 0, NULL) == 1
    # empty batch is a no-op
    assert lib.pa_decode(NULL, NULL, NULL, NULL, d, NULL, 4, NULL, 0, 4, 0.1, 32, 0, NULL, 0, NULL) == 0


def test_prefill_argument_checks(lib):
    assert lib.pa_prefill(FAKE, FAKE, FAKE, FAKE, desc(d=64), FAKE, 4, FAKE, FAKE, 2, 4, 8, 4, 0.1,
                          NULL) == 2
    assert lib.pa_prefill(FAKE, FAKE, FAKE, FAKE, desc(), FAKE, 4, FAKE, FAKE, 2, 3, 8, 4, 0.1,
                          NULL) == 1
    assert lib.pa_prefill(NULL, FAKE, FAKE, FAKE, desc(), FAKE, 4, FAKE, FAKE, 2, 4, 8, 4, 0.1,
                          NULL) == 1
    assert lib.pa_prefill(NULL, NULL, NULL, NULL, desc(), NULL, 4, NULL, NULL, 2, 4, 0, 0, 0.1,
                          NULL) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    k = torch.zeros(4, 2, 128, dtype=torch.bfloat16)
    cache = torch.zeros(16, 16, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_store_kvcache(k, k, cache, cache, torch.zeros(4, dtype=torch.int32))


def test_missing_library_fails_loudly(tmp_path):
    import importlib
    saved = pa._lib
    try:
        pa._lib = None
        with pytest.raises(ImportError, match="no CPU fallback"):
            pa.load_library(str(tmp_path / "nope.so"))
    finally:
        pa._lib = saved


def test_store_decode_argument_checks(lib):
    d = desc(hkv=2)
    ws = FAKE
    # the new rows are required (and 16-byte aligned) when there are sequences
    assert lib.pa_store_decode(NULL, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 4, 0.1,
                               32, 0, ws, 1 << 20, NULL) == 1
    assert lib.pa_store_decode(FAKE, FAKE, NULL, FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 4, 0.1,
                               32, 0, ws, 1 << 20, NULL) == 1
    misaligned = ctypes.c_void_p((1 << 20) + 8)
    assert lib.pa_store_decode(misaligned, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 4,
                               0.1, 32, 0, ws, 1 << 20, NULL) == 1
    # the decode checks still apply: Hq not a multiple of Hkv
    assert lib.pa_store_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 3, 0.1,
                               32, 0, ws, 1 << 20, NULL) == 1
    # empty batch is a no-op
    assert lib.pa_store_decode(NULL, NULL, NULL, NULL, NULL, NULL, NULL, d, NULL, 4, NULL, 0, 4, 0.1,
                               32, 0, NULL, 0, NULL) == 0


def test_binding_store_decode_shapes():
    import torch
    k = torch.zeros(4, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_store_decode(k, k, torch.zeros(4, dtype=torch.int32), k, k, k, k,
                           torch.zeros(4, 4, dtype=torch.int32), torch.zeros(4, dtype=torch.int32),
                           0.1, 32)


def test_copy_blocks_argument_checks(lib):
    d = desc()
    assert lib.pa_copy_blocks(FAKE, FAKE, d, FAKE, FAKE, -1, NULL) == 1
    assert lib.pa_copy_blocks(NULL, FAKE, d, FAKE, FAKE, 2, NULL) == 1
    assert lib.pa_copy_blocks(FAKE, FAKE, d, NULL, FAKE, 2, NULL) == 1
    assert lib.pa_copy_blocks(FAKE, FAKE, desc(bs=12), FAKE, FAKE, 2, NULL) == 1
    assert lib.pa_copy_blocks(NULL, NULL, d, NULL, NULL, 0, NULL) == 0   # no-op


def test_fp8_store_argument_checks(lib):
    d = desc()
    misaligned = ctypes.c_void_p((1 << 20) + 4)
    assert lib.pa_store_kvcache_fp8(FAKE, FAKE, FAKE, FAKE, NULL, FAKE, d, FAKE, 4, NULL) == 1
    assert lib.pa_store_kvcache_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, misaligned, d, FAKE, 4, NULL) == 1
    assert lib.pa_store_kvcache_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, desc(d=96), FAKE, 4, NULL) == 1
    assert lib.pa_store_kvcache_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, d, FAKE, -1, NULL) == 1
    assert lib.pa_store_kvcache_fp8(NULL, NULL, NULL, NULL, NULL, NULL, d, NULL, 0, NULL) == 0


def test_fp8_decode_argument_checks(lib):
    ws = FAKE
    d = desc(hkv=2)
    # both scale arrays are required
    assert lib.pa_decode_fp8(FAKE, FAKE, FAKE, FAKE, NULL, FAKE, d, FAKE, 4, FAKE, 2, 4, 0.1, 32, 128,
                             ws, 1 << 20, NULL) == 1
    # only the tensor-core path reads e4m3 pools: head dim 64 and partitions that are
    # not a multiple of 128 are valid but not implemented
    assert lib.pa_decode_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, desc(hkv=2, d=64), FAKE, 4, FAKE, 2, 4,
                             0.1, 32, 128, ws, 1 << 20, NULL) == 2
    assert lib.pa_decode_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 4, 0.1, 32, 192,
                             ws, 1 << 20, NULL) == 2
    # the decode checks still apply: Hq not a multiple of Hkv
    assert lib.pa_decode_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, d, FAKE, 4, FAKE, 2, 3, 0.1, 32, 128,
                             ws, 1 << 20, NULL) == 1
    assert lib.pa_decode_fp8(NULL, NULL, NULL, NULL, FAKE, FAKE, d, NULL, 4, NULL, 0, 4, 0.1, 32, 0,
                             NULL, 0, NULL) == 0


def test_binding_fp8_checks_pool_shapes():
    import torch
    k = torch.zeros(4, 2, 128, dtype=torch.bfloat16)
    codes = torch.zeros(16, 16, 2, 128, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        pa.pa_store_kvcache_fp8(k, k, codes, codes, torch.zeros(2, 256), torch.zeros(2, 256),
                                torch.zeros(4, dtype=torch.int32))


def test_bench_counter_block_matches_the_library(lib):
    """The graph-replay path clears the workspace's counter block; its size in the
    benchmark must be the library's (the workspace size when nothing is split)."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from workloads import CONFIGS, generate
    w = generate(CONFIGS["tiny_decode"])
    for B, Hq in ((w.num_seqs, w.num_q_heads), (64, 16), (512, 32), (1, 1)):
        w.num_seqs, w.num_q_heads = B, Hq
        assert bench.decode_counter_bytes(w) == pa.pa_decode_workspace_size(B, Hq, 128, 256, 256)
