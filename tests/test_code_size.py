"""The persistent decode kernel's code stays small enough for the SM's instruction caches.

Every SM sub-partition of the decode kernel runs three roles' code (a softmax warp, an
epilogue warp and the producer, issuer or scheduler warp, because the tensor-memory
lane quadrants tie the softmax and epilogue warps to all four sub-partitions). When
the kernel was 96-108 KB of code the per-SM instruction cache hit 78-88% of its
requests and every role's step waited for its instructions; rolled runtime-bounded
loops and out-of-line slow paths of the bounded waits brought it to 67-76 KB and the
e4m3 decode from 81 to 71 us. This test compiles the kernel source (no GPU) and reads
the size of each kernel's code section from the ELF section table, so that a change
that unrolls a runtime loop or inlines a cold path again fails here.
"""
import os
import re
import shutil
import subprocess

import pytest

from paged_kv_cache_442_b200 import build as pa_build

# bytes of code per instantiation (query heads per kv head, e4m3 pools): the current
# sizes plus ~15% headroom
LIMITS = {(2, 0): 78 * 1024, (2, 1): 88 * 1024, (4, 0): 92 * 1024, (4, 1): 108 * 1024}


def _section_sizes(cubin):
    out = subprocess.run(["readelf", "-S", "-W", cubin], capture_output=True, text=True,
                         check=True).stdout
    sizes = {}
    for line in out.splitlines():
        m = re.search(r"\]\s+\.text\.(\S+)\s+\S+\s+\S+\s+\S+\s+([0-9a-f]+)", line)
        if not m:
            continue
        k = re.search(r"decode_tc_kernelILi(\d+)ELb(\d)E", m.group(1))
        if k:
            sizes[(int(k.group(1)), int(k.group(2)))] = int(m.group(2), 16)
    return sizes


def test_decode_kernel_code_fits(tmp_path):
    if shutil.which("readelf") is None:
        pytest.skip("readelf (binutils) not installed")
    try:
        nvcc = pa_build._nvcc()
    except RuntimeError:
        pytest.skip("nvcc not installed")
    cubin = str(tmp_path / "decode_tc.cubin")
    subprocess.run([nvcc, "-O3", "-std=c++17", *pa_build.ARCH, "--expt-relaxed-constexpr",
                    "-I", pa_build.INCLUDE, "-I", pa_build.CSRC, "-cubin",
                    os.path.join(pa_build.CSRC, "decode_tc.cu"), "-o", cubin],
                   check=True, capture_output=True)
    sizes = _section_sizes(cubin)
    assert set(LIMITS) <= set(sizes), sorted(sizes)
    over = {k: (sizes[k], lim) for k, lim in LIMITS.items() if sizes[k] > lim}
    assert not over, f"decode kernel code grew past its budget (bytes, limit): {over}"
