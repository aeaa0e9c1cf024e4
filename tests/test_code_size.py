"""The tensor-core kernels' code stays small enough for the SM's instruction caches.

Every SM sub-partition of the persistent decode kernel runs three roles' code (a
softmax warp, an epilogue warp and the producer, issuer or scheduler warp, because the
tensor-memory lane quadrants tie the softmax and epilogue warps to all four
sub-partitions). When that kernel was 96-108 KB of code the per-SM instruction cache hit
78-88% of its requests and every role's step waited for its instructions; rolled
runtime-bounded loops and out-of-line slow paths of the bounded waits brought it to
67-77 KB and the e4m3 decode from 81 to 71 us (the prefill and shared-prefix kernels,
with the same roles, gained 2-12%). These tests compile the kernel sources (no GPU)
and read the size of each kernel's code section from the ELF section table, so that a
change that unrolls a runtime loop or inlines a cold path again fails here. Budgets
are the current sizes plus ~15%.
"""
import os
import re
import shutil
import subprocess

import pytest

from paged_kv_cache_442_b200 import build as pa_build


def _code_sizes(tmp_path, source, kernel_pattern):
    """{template arguments (or the kernel name): bytes of code} for one source file."""
    if shutil.which("readelf") is None:
        pytest.skip("readelf (binutils) not installed")
    try:
        nvcc = pa_build._nvcc()
    except RuntimeError:
        pytest.skip("nvcc not installed")
    cubin = str(tmp_path / (source + ".cubin"))
    subprocess.run([nvcc, "-O3", "-std=c++17", *pa_build.ARCH, "--expt-relaxed-constexpr",
                    "-I", pa_build.INCLUDE, "-I", pa_build.CSRC, "-cubin",
                    os.path.join(pa_build.CSRC, source), "-o", cubin],
                   check=True, capture_output=True)
    out = subprocess.run(["readelf", "-S", "-W", cubin], capture_output=True, text=True,
                         check=True).stdout
    sizes = {}
    for line in out.splitlines():
        m = re.search(r"\]\s+\.text\.(\S+)\s+\S+\s+\S+\s+\S+\s+([0-9a-f]+)", line)
        if not m:
            continue
        k = re.search(kernel_pattern, m.group(1))
        if k:
            sizes[k.groups() or (k.group(0),)] = int(m.group(2), 16)
    return sizes


def _check(sizes, limits, what):
    assert set(limits) <= set(sizes), (what, sorted(sizes))
    over = {k: (sizes[k], lim) for k, lim in limits.items() if sizes[k] > lim}
    assert not over, f"{what}: code grew past its budget (bytes, limit): {over}"


def test_decode_kernel_code_fits(tmp_path):
    # (query heads per kv head, e4m3 pools)
    sizes = _code_sizes(tmp_path, "decode_tc.cu", r"decode_tc_kernelILi(\d+)ELb(\d)E")
    limits = {("2", "0"): 78 * 1024, ("2", "1"): 88 * 1024, ("4", "0"): 92 * 1024,
              ("4", "1"): 108 * 1024}
    _check(sizes, limits, "decode_tc_kernel")


def test_prefill_kernel_code_fits(tmp_path):
    # (positive scale: the row max taken on the raw scores; new rows stored by the launch)
    sizes = _code_sizes(tmp_path, "prefill.cu", r"prefill_kernelILb(\d)ELb(\d)E")
    limits = {("0", "0"): 84 * 1024, ("1", "0"): 81 * 1024, ("0", "1"): 97 * 1024,
              ("1", "1"): 94 * 1024}
    _check(sizes, limits, "prefill_kernel")


def test_shared_prefix_kernel_code_fits(tmp_path):
    sizes = _code_sizes(tmp_path, "prefix_decode.cu", r"shared_prefix_kernel")
    _check(sizes, {("shared_prefix_kernel",): 70 * 1024}, "shared_prefix_kernel")
