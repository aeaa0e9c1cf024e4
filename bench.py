#!/usr/bin/env python
"""Benchmark of the B200 paged KV-cache hot path.

Headline workload (one "step"): the decode-batch-64 configuration — the 64 new
tokens' K/V rows stored through the slot mapping, then paged decode attention of the
64 sequences (16 q heads / 8 kv heads, head dim 128, block size 256, contexts
uniform in [512, 4096]) — with the whole pool resident in HBM. The step is one
pa_store_decode call (one launch: the decode kernel stores the rows it is about to
read); --separate-store times pa_store_kvcache + pa_decode instead.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0). Under torchrun every rank runs its own batch of the
same shape (independent sequences, no collective): weak scaling, value = all
ranks' bytes / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, SENTINEL_BF16, copy_on_write_append, generate  # noqa: E402

METRIC = ("paged-attn decode achieved HBM GB/s (% of B200 peak); "
          "decode steps/s at batch 64")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
DATASHEET_HBM_GBS = 8000.0
L2_FLUSH_BYTES = 256 << 20


# --------------------------------------------------------------------------- utils
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), \
            float(d.get("bf16_tflops_sustained", d.get("bf16_tflops", FALLBACK_BF16_TFLOPS))), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def file_hash(*paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


DECODE_SRC = ("paged_kv_cache_442_b200/csrc/decode.cu", "paged_kv_cache_442_b200/csrc/decode_tc.cu",
              "paged_kv_cache_442_b200/csrc/pa_api.cu", "paged_kv_cache_442_b200/csrc/pa_ptx.cuh")
PREFILL_SRC = ("paged_kv_cache_442_b200/csrc/prefill.cu", "paged_kv_cache_442_b200/csrc/pa_ptx.cuh")


def recorded_traffic(name, srcs):
    """Per-launch DRAM bytes from a committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", f"{name}.traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_hash") != file_hash(*srcs):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while a region runs."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0=None, t1=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ts, line in self.lines:
            if t0 is not None and not (t0 - 0.06 <= ts <= t1 + 0.06):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[3:7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples in timed region"],
                    "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- byte/flop counts
def decode_bytes(w):
    """Algorithmic bytes of one decode: K/V rows of every visible position, q, out."""
    kv = int(w.context_lens.astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * 2 * 2
    qo = 2 * w.num_seqs * w.num_q_heads * w.head_dim * 2
    return kv + qo


def store_bytes(w):
    """new k/v read + written once each."""
    return 2 * 2 * len(w.new_slots) * w.num_kv_heads * w.head_dim * 2


def prefill_flops(w):
    """Causal-exact: 4*D flops per (query, head, visible key)."""
    tot = 0
    for s in range(w.num_seqs):
        n = int(w.new_lens[s])
        ctx = int(w.context_lens[s])
        first = ctx - n
        # sum over i of (first + i + 1)
        tot += n * (first + 1) + n * (n - 1) // 2
    return 4 * w.head_dim * w.num_q_heads * tot


def prefill_bytes(w):
    kv = int(w.context_lens.astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * 2 * 2
    qo = 2 * int(w.new_lens.sum()) * w.num_q_heads * w.head_dim * 2
    return kv + qo


# --------------------------------------------------------------------------- GPU arm
class GpuRunner:
    def __init__(self, w, torch, pa, partition_size=0, separate_store=False, cow=None,
                 shared_len=0):
        self.w, self.torch, self.pa = w, torch, pa
        self.shared_len = shared_len
        dev = torch.device("cuda")
        shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
        fill = int(np.uint16(SENTINEL_BF16).view(np.int16))
        self.k_cache = torch.full(shape, fill, dtype=torch.int16, device=dev).view(torch.bfloat16)
        self.v_cache = torch.full(shape, fill, dtype=torch.int16, device=dev).view(torch.bfloat16)

        def bf(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

        def i32(a):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)

        if len(w.setup_slots):
            # untimed setup: the cached context, written in chunks through the library
            n = len(w.setup_slots)
            step = 1 << 18
            for s0 in range(0, n, step):
                idx = np.arange(s0, min(n, s0 + step))
                pa.pa_store_kvcache(bf(w.src_k[w.setup_src[idx]]), bf(w.src_v[w.setup_src[idx]]),
                                    self.k_cache, self.v_cache, i32(w.setup_slots[idx]))
        self.q = bf(w.q)
        self.new_k = bf(w.new_k) if len(w.new_slots) else None
        self.new_v = bf(w.new_v) if len(w.new_slots) else None
        self.new_slots = i32(w.new_slots)
        self.block_tables = i32(w.block_tables)
        self.context_lens = i32(w.context_lens)
        self.cu = i32(w.cu_seqlens_q)
        self.out = torch.empty_like(self.q)
        if w.kind == "decode" and shared_len:
            # the shared prefix attended once (its blocks: the longest sequence's first
            # ones, held by every sequence), then the rest of every context
            s_long = int(np.argmax(w.context_lens))
            self.shared_blocks = i32(w.block_tables[s_long, :shared_len // w.block_size])
            self.ws, self.P = pa.shared_prefix_workspace(
                w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.max_context_len,
                shared_len, partition_size)
        elif w.kind == "decode":
            self.ws, self.P = pa.decode_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads,
                                                  w.head_dim, w.max_context_len, partition_size)
        tc = False
        if w.kind == "decode":
            # kernels one pa_decode launches: the persistent tcgen05 kernel merges its
            # partitions itself (head dim 128, partition a multiple of 128 up to 2048);
            # the CUDA-core kernel adds a reduce launch when the context is split
            G = w.num_q_heads // w.num_kv_heads
            tc = (w.head_dim == 128 and G in (1, 2, 4, 8, 16) and self.P % 128 == 0
                  and self.P <= 2048)
            split = self.P < w.max_context_len
            self.decode_launches = 1 if tc or not split else 2
            if shared_len:
                self.decode_launches = 2 if w.max_context_len > shared_len else 1
        # a step that stores new tokens runs as one pa_store_decode / pa_store_prefill
        # call (the kernel stores the rows itself; decode shapes off the tensor-core
        # path add a store launch)
        self.fused = self.new_k is not None and not separate_store
        # copy-on-write pairs copied before each step (blocks the step appends into)
        self.cow = None if cow is None else (i32(cow[0]), i32(cow[1]))
        if self.fused and w.kind == "decode" and not tc:
            self.decode_launches += 1
        self.max_q = int(np.max(np.diff(w.cu_seqlens_q))) if w.num_seqs else 0
        torch.cuda.synchronize()

    def store(self, k=None, v=None, slots=None):
        if self.cow is not None:
            self.pa.pa_copy_blocks(self.k_cache, self.v_cache, *self.cow)
            if self.fused:
                return 1
        if self.fused or (self.new_k is None and k is None):
            return 1 if self.cow is not None else 0
        self.pa.pa_store_kvcache(self.new_k if k is None else k, self.new_v if v is None else v,
                                 self.k_cache, self.v_cache, self.new_slots if slots is None else slots)
        return 1

    def attend(self, q=None, ctx=None, bt=None, out=None, k=None, v=None, slots=None):
        w, pa = self.w, self.pa
        q = self.q if q is None else q
        out = self.out if out is None else out
        ctx = self.context_lens if ctx is None else ctx
        bt = self.block_tables if bt is None else bt
        if self.fused and w.kind == "decode":
            pa.pa_store_decode(self.new_k if k is None else k, self.new_v if v is None else v,
                               self.new_slots if slots is None else slots, out, q, self.k_cache,
                               self.v_cache, bt, ctx, w.scale, w.max_context_len, self.P, self.ws)
            return self.decode_launches
        if self.fused:
            pa.pa_store_prefill(self.new_k if k is None else k, self.new_v if v is None else v,
                                self.new_slots if slots is None else slots, out, q, self.k_cache,
                                self.v_cache, bt, self.cu, ctx, w.scale, self.max_q)
            return 1
        if w.kind == "decode" and self.shared_len:
            pa.pa_decode_shared_prefix(out, q, self.k_cache, self.v_cache, bt, ctx, w.scale,
                                       w.max_context_len, self.shared_blocks, self.shared_len,
                                       self.P, self.ws)
            return self.decode_launches
        if w.kind == "decode":
            pa.pa_decode(out, q, self.k_cache, self.v_cache, bt, ctx, w.scale,
                         w.max_context_len, self.P, self.ws)
            return self.decode_launches
        pa.pa_prefill(out, q, self.k_cache, self.v_cache, bt, self.cu, ctx, w.scale, self.max_q)
        return 1

    def step(self):
        return self.store() + self.attend()


def fp8_decode_bytes(w):
    """Bytes an fp8 decode reads and writes: the e4m3 codes and the fp32 row scales of K
    and V at every position of every sequence, q in and the output out."""
    pos = int(w.context_lens.astype(np.int64).sum())
    kv = pos * w.num_kv_heads * (w.head_dim + 4) * 2
    qo = 2 * w.num_seqs * w.num_q_heads * w.head_dim * 2
    return kv + qo


def fp8_store_bytes(w):
    """Bytes the fp8 store moves: bf16 rows in, codes and scales out (K and V)."""
    return len(w.new_slots) * w.num_kv_heads * (2 * w.head_dim + w.head_dim + 4) * 2


class Fp8Runner:
    """A decode step over e4m3 pools: the step's new rows quantised into the pools
    (pa_store_kvcache_fp8), then pa_decode_fp8. The cached context is quantised by the
    same store during setup (untimed); unwritten rows hold NaN codes and scales."""

    def __init__(self, w, torch, pa):
        self.w, self.pa = w, pa
        dev = torch.device("cuda")
        shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
        self.k8 = torch.full(shape, 0x7F, dtype=torch.uint8, device=dev)
        self.v8 = torch.full(shape, 0x7F, dtype=torch.uint8, device=dev)
        sshape = (w.num_kv_heads, w.num_blocks * w.block_size)
        self.ks = torch.full(sshape, float("nan"), dtype=torch.float32, device=dev)
        self.vs = torch.full(sshape, float("nan"), dtype=torch.float32, device=dev)

        def bf(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

        def i32(a):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)

        n = len(w.setup_slots)
        for s0 in range(0, n, 1 << 18):
            idx = np.arange(s0, min(n, s0 + (1 << 18)))
            pa.pa_store_kvcache_fp8(bf(w.src_k[w.setup_src[idx]]), bf(w.src_v[w.setup_src[idx]]),
                                    self.k8, self.v8, self.ks, self.vs, i32(w.setup_slots[idx]))
        self.q = bf(w.q)
        self.new_k = bf(w.new_k) if len(w.new_slots) else None
        self.new_v = bf(w.new_v) if len(w.new_slots) else None
        self.new_slots = i32(w.new_slots)
        self.block_tables = i32(w.block_tables)
        self.context_lens = i32(w.context_lens)
        self.out = torch.empty_like(self.q)
        self.ws, self.P = pa.decode_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads,
                                              w.head_dim, w.max_context_len)
        torch.cuda.synchronize()

    def store(self):
        if self.new_k is None:
            return 0
        self.pa.pa_store_kvcache_fp8(self.new_k, self.new_v, self.k8, self.v8, self.ks, self.vs,
                                     self.new_slots)
        return 1

    def attend(self):
        w = self.w
        self.pa.pa_decode_fp8(self.out, self.q, self.k8, self.v8, self.ks, self.vs,
                              self.block_tables, self.context_lens, w.scale, w.max_context_len,
                              self.P, self.ws)
        return 1

    def step(self):
        return self.store() + self.attend()


def measure_fp8_decode(torch, pa, hbm_peak, peak_src, bf16_attn_us, steps=200, warmup=10):
    """The headline decode batch over e4m3 pools (same sequences, same step shape)."""
    w = generate(CONFIGS["decode_b64"])
    r = Fp8Runner(w, torch, pa)
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    total_ms, attn_ms, lps = time_steps(r, torch, steps, warmup, flush)
    a_ms = sum(attn_ms) / len(attn_ms)
    st_ms = total_ms / steps - a_ms
    b = fp8_decode_bytes(w)
    d = {"kernel": "pa_decode_fp8 (persistent tcgen05 decode; kind::f8f6f4 MMAs read the "
                   "stored e4m3 codes, row scales applied in the softmax)",
         "attn_us": round(a_ms * 1e3, 2),
         "step_us": round(total_ms / steps * 1e3, 2), "steps": steps, "launches_per_step": lps,
         "algorithmic_bytes": b, "GBps": round(b / a_ms / 1e6, 1),
         "frac_of_hbm_peak": round(b / a_ms / 1e6 / hbm_peak, 3),
         "store_us": round(st_ms * 1e3, 2),
         "store_GBps": round(fp8_store_bytes(w) / st_ms / 1e6, 1) if st_ms > 0 else None,
         "partition_size": r.P, "peak_source": peak_src}
    if bf16_attn_us:
        d["attn_time_vs_bf16_store_decode"] = round(a_ms * 1e3 / bf16_attn_us, 3)
    del r
    torch.cuda.empty_cache()
    return d


def time_steps(runner, torch, steps, warmup, flush_buf, barrier=None):
    """Per-step device time (ms) of `steps` steps, L2 flushed before each step.

    Returns (total step ms, attention-call ms list, launches per step)."""
    stream = torch.cuda.current_stream()
    flush_out = torch.zeros((), dtype=flush_buf.dtype, device=flush_buf.device)
    for _ in range(warmup):
        torch.sum(flush_buf, dim=0, out=flush_out)
        runner.step()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    launches = 0
    for i in range(steps):
        torch.sum(flush_buf, dim=0, out=flush_out)     # read 256 MiB: evicts the previous step from L2
        a, b, c = ev[i]
        a.record(stream)
        launches += runner.store()
        b.record(stream)
        launches += runner.attend()
        c.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    attn_ms = [b.elapsed_time(c) for _, b, c in ev]
    return sum(step_ms), attn_ms, launches // steps


def decode_counter_bytes(w):
    """The leading block of the decode workspace that holds the tagged work and arrival
    counters (include/pa.h, pa_decode_workspace_size)."""
    return -(-(8 * (1 + w.num_seqs * w.num_q_heads)) // 256) * 256


def time_graph(runner, torch, steps, warmup, flush_buf):
    """The decode step replayed from a CUDA graph (launch overhead out of the picture).

    A captured call keeps the counter tag it was captured with, so the graph first
    clears the workspace's counter block (a replay is then a fresh call). Returns
    (mean step us, whether the replayed output equals the eager output bit for bit),
    or an error string."""
    try:
        w = runner.w
        n = decode_counter_bytes(w) // 4
        runner.step()
        torch.cuda.synchronize()
        eager = runner.out.clone()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(2):
                runner.ws[:n].zero_()
                runner.step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            runner.ws[:n].zero_()
            runner.step()
        runner.out.zero_()
        flush_out = torch.zeros((), dtype=flush_buf.dtype, device=flush_buf.device)
        for _ in range(warmup):
            torch.sum(flush_buf, dim=0, out=flush_out)
            g.replay()
        torch.cuda.synchronize()
        same = bool(torch.equal(runner.out.view(torch.int16), eager.view(torch.int16)))
        stream = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            torch.sum(flush_buf, dim=0, out=flush_out)
            ev[i][0].record(stream)
            g.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        us = sum(a.elapsed_time(b) for a, b in ev) / steps * 1e3
        del g
        return round(us, 2), same
    except Exception as e:  # noqa: BLE001  (reported, not fatal to the run)
        return None, f"{type(e).__name__}: {e}"


class PackedInputs:
    """One step's host inputs packed into a single pinned buffer (q, new K/V rows,
    slots, context lengths, block tables; each piece on a 256-byte boundary) and a
    device buffer of the same layout whose typed views the library call takes, so a
    step's inputs cross PCIe in ONE host-to-device copy and its output in one
    device-to-host copy."""

    def __init__(self, runner, torch):
        pieces = [("q", runner.q), ("k", runner.new_k), ("v", runner.new_v),
                  ("slots", runner.new_slots), ("ctx", runner.context_lens),
                  ("bt", runner.block_tables)]
        self.layout, off = {}, 0
        for name, t in pieces:
            if t is None or t.numel() == 0:
                continue
            n = t.numel() * t.element_size()
            self.layout[name] = (off, n, t.dtype, tuple(t.shape))
            off += -(-n // 256) * 256
        self.nbytes = off
        self.host = torch.empty(off, dtype=torch.uint8).pin_memory()
        for name, t in pieces:
            if t is not None and name in self.layout:
                o, n, _, _ = self.layout[name]
                self.host[o:o + n].copy_(t.contiguous().view(torch.uint8).view(-1).cpu())
        self.torch = torch

    def device_views(self, dev_buf):
        views = {}
        for name, (o, n, dt, shape) in self.layout.items():
            views[name] = dev_buf[o:o + n].view(dt).view(shape)
        return views


def time_e2e(runner, torch, steps, warmup):
    """The step through the host, as a caller without device-resident inputs runs it:
    every step copies its packed inputs from pinned host memory to the device (one
    copy), makes the library call on them, and copies the output back (one copy), all
    in order on one stream. Returns (total ms, h2d bytes, d2h bytes, pipelined ms):
    the last is the same steps with two buffer sets, the copies on a second stream
    overlapping the previous step's kernel (a serving loop's steady state)."""
    pk = PackedInputs(runner, torch)
    d_in = torch.empty(pk.nbytes, dtype=torch.uint8, device="cuda")
    v = pk.device_views(d_in)
    d_out = torch.empty_like(runner.out)
    h_out = torch.empty(runner.out.shape, dtype=runner.out.dtype).pin_memory()
    h2d = pk.nbytes
    d2h = h_out.numel() * h_out.element_size()

    def one(views, dout, hout, copy_stream=None):
        d = views
        slots = d.get("slots", runner.new_slots)   # an empty slot list is not copied
        runner.store(d.get("k"), d.get("v"), slots)
        runner.attend(d["q"], d["ctx"], d["bt"], dout, d.get("k"), d.get("v"), slots)

    def serial():
        d_in.copy_(pk.host, non_blocking=True)
        one(v, d_out, h_out)
        h_out.copy_(d_out, non_blocking=True)

    for _ in range(warmup):
        serial()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        serial()
    e.record()
    torch.cuda.synchronize()
    serial_ms = s.elapsed_time(e)
    if not torch.equal(h_out.view(torch.int16), runner.out.cpu().view(torch.int16)):
        # the step is deterministic: the copied-back output must be the device one
        raise RuntimeError("end-to-end output differs from the device-resident step")

    # pipelined: buffer set i % 2; step i's input copy overlaps step i-1's kernel and
    # step i-1's output copy overlaps step i's kernel. One stream per copy direction
    # (the two directions have their own copy engines): on a single copy stream the
    # input copy of step i would queue behind the output copy of step i-1, which waits
    # for kernel i-1, and nothing would overlap.
    main = torch.cuda.current_stream()
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = [(torch.empty(pk.nbytes, dtype=torch.uint8, device="cuda"), torch.empty_like(runner.out),
             torch.empty(runner.out.shape, dtype=runner.out.dtype).pin_memory()) for _ in range(2)]
    views = [pk.device_views(b[0]) for b in bufs]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_k = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def pipelined(n):
        for i in range(n):
            b = i % 2
            din, dout, hout = bufs[b]
            with torch.cuda.stream(hs):
                if i >= 2:
                    hs.wait_event(ev_k[b])       # the kernel of step i-2 read this buffer
                din.copy_(pk.host, non_blocking=True)
                ev_in[b].record(hs)
            main.wait_event(ev_in[b])
            if i >= 2:
                main.wait_event(ev_out[b])       # step i-2's output has been copied out
            one(views[b], dout, hout)
            ev_k[b].record(main)
            with torch.cuda.stream(ds):
                ds.wait_event(ev_k[b])
                hout.copy_(dout, non_blocking=True)
                ev_out[b].record(ds)
        main.wait_stream(hs)
        main.wait_stream(ds)

    pipelined(warmup)
    torch.cuda.synchronize()
    s.record(main)
    hs.wait_event(s)
    ds.wait_event(s)
    pipelined(steps)
    e.record(main)
    torch.cuda.synchronize()
    for _, dout, hout in bufs:
        if not torch.equal(hout.view(torch.int16), runner.out.cpu().view(torch.int16)):
            raise RuntimeError("pipelined end-to-end output differs from the device-resident step")
    return serial_ms, h2d, d2h, s.elapsed_time(e)


# --------------------------------------------------------------------------- CPU (oracle) arm
def oracle_pools_for(w):
    """The oracle's own pools: setup rows and this step's new rows, stored by the oracle."""
    import oracle
    kc, vc = w.empty_pool(), w.empty_pool()
    if len(w.setup_slots):
        kc, vc = oracle.store_kvcache(kc, vc, w.setup_k, w.setup_v, w.setup_slots)
    if len(w.new_slots):
        kc, vc = oracle.store_kvcache(kc, vc, w.new_k, w.new_v, w.new_slots)
    return kc, vc


def oracle_decode_one(w, pools, s):
    """Oracle decode of sequence s; returns (seconds, algorithmic bytes)."""
    import oracle
    kc, vc = pools
    idx = np.array([s])
    t0 = time.perf_counter()
    oracle.decode(w.q[idx], kc, vc, w.block_tables[idx], w.context_lens[idx], w.scale)
    dt = time.perf_counter() - t0
    nbytes = int(w.context_lens[s]) * w.num_kv_heads * w.head_dim * 4 + 2 * w.num_q_heads * w.head_dim * 2
    return dt, nbytes


def host_threads():
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        blas = cores
    return cores, blas


def cpu_oracle_time(w, budget_s=12.0, pools=None):
    """The oracle (as it stands) decoding sequences one at a time for ~budget_s.

    Returns (seconds, bytes, sequences decoded, cores, blas threads)."""
    pools = oracle_pools_for(w) if pools is None else pools
    tot_t, tot_b, n = 0.0, 0, 0
    while tot_t < budget_s:
        dt, nb = oracle_decode_one(w, pools, n % w.num_seqs)
        tot_t += dt
        tot_b += nb
        n += 1
    cores, blas = host_threads()
    return tot_t, tot_b, n, cores, blas


def cpu_oracle_time_one_core(w, budget_s=4.0):
    """The same oracle with its BLAS limited to one thread (GB/s, sequences decoded)."""
    try:
        from threadpoolctl import threadpool_limits
    except Exception:  # noqa: BLE001
        return None, 0
    with threadpool_limits(limits=1):
        t, b, n, _, _ = cpu_oracle_time(w, budget_s)
    return b / t / 1e9, n


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_b64")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the extra per-configuration measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--partition-size", type=int, default=0)
    ap.add_argument("--separate-store", action="store_true",
                    help="decode steps as pa_store_kvcache + pa_decode instead of pa_store_decode")
    ap.add_argument("--fp8-only", action="store_true",
                    help="print only the decode-batch-64 step over e4m3 pools (one GPU)")
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="the configuration's first N sequences only (a small case for "
                         "profiling; not a headline number)")
    ap.add_argument("--shared-prefix", action="store_true",
                    help="decode the workload's shared prefix once for all sequences "
                         "(pa_decode_shared_prefix; prefix-sharing workloads)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.fp8_only and int(os.environ.get("WORLD_SIZE", "1")) > 1:
        ap.error("--fp8-only runs on one GPU")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = CONFIGS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return
        run_reference(args, cfg, world)
        return

    import torch
    import paged_kv_cache_442_b200 as pa
    torch.cuda.set_device(local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    hbm_peak, tf_peak, tf_sustained, peak_src = peaks()
    if args.fp8_only:
        if rank == 0:
            print(json.dumps({"decode_b64_fp8": measure_fp8_decode(
                torch, pa, hbm_peak, peak_src, None, steps=args.steps, warmup=args.warmup)}),
                flush=True)
        return
    # every rank decodes its own batch of the same shape (weak scaling)
    w = rank_workload(cfg, rank, args.num_seqs)
    shared = cfg.shared_prefix_len if args.shared_prefix else 0
    runner = GpuRunner(w, torch, pa, args.partition_size, args.separate_store, shared_len=shared)
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    t0 = time.time()
    total_ms, attn_ms, launches_per_step = time_steps(runner, torch, args.steps, args.warmup, flush,
                                                      barrier)
    t1 = time.time()
    clocks = sampler.stop(t0, t1)

    step_ms = max_over_ranks(total_ms / args.steps, pg, torch, "cuda")
    bytes_step = (decode_bytes(w) if w.kind == "decode" else prefill_bytes(w)) + store_bytes(w)
    unique = None
    if shared:
        # the shared prefix is read once for all sequences: the bytes the step must move
        # are the unique ones (every distinct K/V row once, q, out)
        unique = w.kv_bytes_unique() + 2 * w.num_seqs * w.num_q_heads * w.head_dim * 2
        bytes_step = unique + store_bytes(w)
    job_bytes = sum_over_ranks(bytes_step, pg, torch, "cuda")
    value = job_gbps(job_bytes, step_ms)
    attn_avg_ms = sum(attn_ms) / len(attn_ms)
    attn_bytes = decode_bytes(w) if w.kind == "decode" else prefill_bytes(w)
    if runner.fused:
        attn_bytes += store_bytes(w)  # the new rows are read and written by the same launch
    if unique is not None:
        attn_bytes = unique
    achieved = attn_bytes / (attn_avg_ms * 1e-3) / 1e9
    if w.kind == "decode":
        kname = ("pa_store_decode (persistent tcgen05 decode; new-row store and split-K merge inside)"
                 if runner.fused else
                 "pa_decode_shared_prefix (dense tcgen05 pass over the shared prefix + persistent "
                 "decode of the rest; time of both launches)" if shared else
                 "pa_decode (persistent tcgen05 decode, split-K merge inside)")
        roofline = {"bound": "hbm", "kernel": kname,
                    "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                    "frac": round(achieved / hbm_peak, 3), "peak_source": f"{peak_src} copy bandwidth",
                    "algorithmic_bytes_per_launch": attn_bytes,
                    "avg_launch_us": round(attn_avg_ms * 1e3, 2),
                    "traffic": recorded_traffic(cfg.name + ".decode", DECODE_SRC)}
    else:
        fl = prefill_flops(w)
        tf = fl / (attn_avg_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": "pa_prefill (tcgen05)", "achieved": round(tf, 1),
                    "peak": tf_peak, "unit": "TFLOP/s", "frac": round(tf / tf_peak, 3),
                    "frac_of_sustained": round(tf / tf_sustained, 3),
                    "peak_source": f"{peak_src} bf16 GEMM (burst)",
                    "algorithmic_flops_per_launch": fl, "avg_launch_us": round(attn_avg_ms * 1e3, 2),
                    "traffic": recorded_traffic(cfg.name + ".prefill", PREFILL_SRC)}

    e2e_ms, h2d, d2h, e2e_pipe_ms = time_e2e(runner, torch, min(args.steps, 500), args.warmup)
    graph = None
    if w.kind == "decode" and not args.headline_only:
        g_us, g_same = time_graph(runner, torch, min(args.steps, 500), args.warmup, flush)
        graph = {"step_us": g_us, "eager_step_us": round(step_ms * 1e3, 2),
                 "output_equals_eager": g_same,
                 "graph": "clear the workspace counter block, then the step's library call"}
    e2e_step_ms = max_over_ranks(e2e_ms / min(args.steps, 500), pg, torch, "cuda")
    e2e_pipe_step_ms = max_over_ranks(e2e_pipe_ms / min(args.steps, 500), pg, torch, "cuda")

    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.name + (f" (first {w.num_seqs} sequences)" if args.num_seqs else "")
                   + (" (shared prefix attended once)" if shared else ""), "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
                   "block_size": w.block_size, "num_blocks": w.num_blocks,
                   "context_lens": f"{cfg.ctx_dist}[{cfg.ctx_lo},{cfg.ctx_hi}] sum={int(w.context_lens.sum())}",
                   "partition_size": getattr(runner, "P", None),
                   "parallelism": f"replicas x{world} (independent batches)",
                   "l2": "flushed before every step by reading a 256 MiB buffer (clean lines; outside the step events)",
                   "bytes": ("unique: every distinct K/V row once (the shared prefix is attended once), q, out"
                             if shared else "every sequence's K/V rows, q, out (+ the new rows when stored)")},
        "steps_per_s": round(1e3 / step_ms * world, 1),
        "pct_of_hbm_peak": round(100 * value / world / hbm_peak, 1),
        "pct_of_datasheet_8tbs": round(100 * value / world / DATASHEET_HBM_GBS, 1),
        "bytes_per_step": bytes_step,
        "roofline": roofline,
        "e2e": {"value": round(job_gbps(job_bytes, e2e_pipe_step_ms), 1), "unit": "GB/s",
                "ms_per_step": round(e2e_pipe_step_ms, 5), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "api": ("paged_kv_cache_442_b200.pa_store_decode" if runner.fused else
                        "paged_kv_cache_442_b200.pa_store_kvcache + pa_decode") +
                       " (C ABI) on pinned host buffers",
                "copies_per_step": "one packed host-to-device copy of all inputs, one "
                                   "device-to-host copy of the output",
                "how": "a serving loop's steady state: two buffer sets, the input copy of "
                       "step i on one stream overlaps kernel i-1, the output copy of step i-1 "
                       "on another overlaps kernel i; every step's output is copied back and "
                       "checked against the device-resident step",
                "serial": {"value": round(job_gbps(job_bytes, e2e_step_ms), 1),
                           "ms_per_step": round(e2e_step_ms, 5),
                           "how": "input copy, library call, output copy in order on one stream"}},
        "gpu_launches": launches_per_step * args.steps,
        "cuda_graph": graph,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.headline_only:
        line["other_workloads"] = measure_others(torch, pa, hbm_peak, tf_peak, tf_sustained, peak_src)
        if cfg.name == "decode_b64":
            line["other_workloads"]["decode_b64_fp8"] = measure_fp8_decode(
                torch, pa, hbm_peak, peak_src, attn_avg_ms * 1e3)
        line["block_manager"] = measure_block_manager(torch, pa)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ct, cb, n, cores, blas = cpu_oracle_time(w)
        line["cpu_baseline"] = {"value": round(cb / ct / 1e9, 4), "unit": "GB/s", "cores": cores,
                                "blas_threads": blas, "kind": "oracle",
                                "sample": f"oracle decode of {n} single sequences of {cfg.name} "
                                          f"on its own pools ({ct:.1f} s of CPU time)"}
        v1, n1 = cpu_oracle_time_one_core(w)
        if v1 is not None:
            line["cpu_baseline"]["value_one_blas_thread"] = round(v1, 4)
            line["cpu_baseline"]["sample_one_blas_thread"] = f"{n1} sequences, ~4 s"
            if not args.headline_only:
                # the one-core oracle on the other decode configurations as well
                one = {}
                for name in ("tiny_decode", "long_ctx_decode"):
                    wo = generate(CONFIGS[name])
                    g1, k1 = cpu_oracle_time_one_core(wo)
                    one[name] = {"GBps": round(g1, 4), "sample": f"{k1} sequences, ~4 s"}
                    del wo
                line["cpu_baseline"]["one_blas_thread_other_configs"] = one
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def rank_workload(cfg, rank, num_seqs=None):
    """Rank r's batch: the same configuration (shape) drawn from another seed, so the
    ranks decode independent sequences (weak scaling; rank 0's batch is the
    configuration's own). num_seqs keeps the first sequences only (profiling)."""
    from dataclasses import replace
    return generate(replace(cfg, index=cfg.index + 100 * rank), num_seqs=num_seqs)


def max_over_ranks(x, dist, torch, device):
    """The slowest rank's value (every rank gets it); x itself when not distributed."""
    if dist is None:
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, dist, torch, device):
    """Sum over ranks (every rank gets it); x itself when not distributed."""
    if dist is None:
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_gbps(job_bytes, step_ms):
    """Whole-job throughput: the bytes all ranks moved in a step over the slowest
    rank's step time."""
    return job_bytes / (step_ms * 1e-3) / 1e9


def measure_others(torch, pa, hbm_peak, tf_peak, tf_sustained, peak_src, steps=200, warmup=10):
    """Device-timed numbers of the other configurations (same method, fewer steps)."""
    res = {}
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    for name in ("long_ctx_decode", "prefix_share_decode", "prefix_share_cow_append",
                 "chunked_prefill"):
        cow = None
        if name == "prefix_share_cow_append":
            # the prefix-sharing batch appending each sequence's token: the shared blocks
            # the sequences append into are copied first, then one pa_store_decode
            w, src, dst = copy_on_write_append(generate(CONFIGS["prefix_share_decode"]))
            cow = (src, dst)
        else:
            w = generate(CONFIGS[name])
        # prefill: the attention kernel alone after a separate store (its roofline),
        # then the step as one pa_store_prefill launch
        r = GpuRunner(w, torch, pa, cow=cow, separate_store=(w.kind == "prefill"))
        n = steps if w.kind == "decode" else 50
        total_ms, attn_ms, lps = time_steps(r, torch, n, warmup, flush)
        a_ms = sum(attn_ms) / len(attn_ms)
        d = {"attn_us": round(a_ms * 1e3, 2), "step_us": round(total_ms / n * 1e3, 2), "steps": n}
        if w.kind == "decode":
            lb = decode_bytes(w) + (store_bytes(w) if r.fused else 0)
            d.update({"kernel": "pa_store_decode" if r.fused else "pa_decode", "logical_bytes": lb, "logical_GBps": round(lb / a_ms / 1e6, 1),
                      "frac_of_hbm_peak_logical": round(lb / a_ms / 1e6 / hbm_peak, 3),
                      "partition_size": r.P})
            if cow is not None:
                # many sequences copy the same few shared prefix blocks: the bytes the
                # copy must move through DRAM are the distinct sources read once and
                # every destination written (K and V)
                blk = w.block_size * w.num_kv_heads * w.head_dim * 2
                moved = 4 * len(cow[0]) * blk
                dram = 2 * (len(np.unique(cow[0])) + len(cow[1])) * blk
                c_ms = total_ms / n - a_ms
                d.update({"copy_pairs": len(cow[0]), "copy_distinct_sources": int(len(np.unique(cow[0]))),
                          "copy_us": round(c_ms * 1e3, 2), "copy_moved_bytes": moved,
                          "copy_dram_bytes": dram, "copy_dram_GBps": round(dram / c_ms / 1e6, 1),
                          "copy_frac_of_hbm_peak": round(dram / c_ms / 1e6 / hbm_peak, 3)})
            if name.startswith("prefix_share"):
                ub = w.kv_bytes_unique() + 2 * w.num_seqs * w.num_q_heads * w.head_dim * 2
                d.update({"unique_bytes": ub, "unique_GBps": round(ub / a_ms / 1e6, 1),
                          "frac_of_hbm_peak_unique": round(ub / a_ms / 1e6 / hbm_peak, 3)})
            if name == "prefix_share_decode":
                # the same batch with its shared prefix attended once for all sequences
                del r
                torch.cuda.empty_cache()
                S = CONFIGS[name].shared_prefix_len
                r = GpuRunner(w, torch, pa, shared_len=S)
                s_ms, s_attn, s_lps = time_steps(r, torch, n, warmup, flush)
                sa = sum(s_attn) / len(s_attn)
                d["shared_prefix"] = {
                    "kernel": "pa_decode_shared_prefix (dense tcgen05 pass over the shared "
                              "prefix + persistent decode of the rest)",
                    "shared_len": S, "attn_us": round(sa * 1e3, 2), "launches": s_lps,
                    "partition_size": r.P,
                    "logical_GBps": round(lb / sa / 1e6, 1),
                    "unique_GBps": round(ub / sa / 1e6, 1),
                    "frac_of_hbm_peak_unique": round(ub / sa / 1e6 / hbm_peak, 3),
                    "speedup_vs_pa_decode": round(a_ms / sa, 3)}
        else:
            fl = prefill_flops(w)
            st_ms = total_ms / n - a_ms
            d.update({"kernel": "pa_prefill (tcgen05)", "flops": fl,
                      "TFLOPs": round(fl / a_ms / 1e9, 1),
                      "frac_of_bf16_peak_sustained": round(fl / a_ms / 1e9 / tf_sustained, 3),
                      "frac_of_bf16_peak_burst": round(fl / a_ms / 1e9 / tf_peak, 3),
                      "store_us": round(st_ms * 1e3, 2),
                      "store_GBps": round(store_bytes(w) / st_ms / 1e6, 1),
                      "separate_store_step_us": round(total_ms / n * 1e3, 2)})
            del r
            torch.cuda.empty_cache()
            r = GpuRunner(w, torch, pa)
            f_ms, f_attn, f_lps = time_steps(r, torch, n, warmup, flush)
            fa = sum(f_attn) / len(f_attn)
            d.update({"step_us": round(f_ms / n * 1e3, 2), "step_launches": f_lps,
                      "step": "one pa_store_prefill launch (new rows stored by the attention "
                              "kernel)",
                      "step_TFLOPs": round(fl / fa / 1e9, 1)})
        d["peak_source"] = peak_src
        res[name] = d
        del r
        torch.cuda.empty_cache()
    return res


def measure_block_manager(torch, pa, reps=50):
    """Prefix-sharing batch (512 requests, lognormal lengths, a shared 1024-token
    prompt, block size 64): the batched GPU block hashes, and the host block manager
    allocating every request's table (hashes given, and hashed on the host)."""
    cfg = CONFIGS["prefix_share_decode"]
    w = generate(cfg)
    rng = np.random.default_rng(11)
    prefix = rng.integers(1, 1 << 20, size=1024).tolist()
    seqs = [prefix[:n] + rng.integers(1, 1 << 20, size=max(0, int(n) - 1024)).tolist()
            for n in w.context_lens]
    bs = cfg.block_size
    lens = np.array([len(x) for x in seqs], dtype=np.int64)
    toks = np.concatenate([np.asarray(x, dtype=np.int32) for x in seqs])
    cu_t = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).cuda()
    cu_b_h = np.concatenate([[0], np.cumsum(lens // bs)]).astype(np.int32)
    cu_b = torch.from_numpy(cu_b_h).cuda()
    d_t = torch.from_numpy(toks).cuda()
    out = torch.zeros(int(cu_b_h[-1]), dtype=torch.int32, device="cuda")
    for _ in range(3):
        pa.pa_block_hashes(d_t, cu_t, cu_b, bs, out)
    torch.cuda.synchronize()
    s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s_ev.record()
    for _ in range(reps):
        pa.pa_block_hashes(d_t, cu_t, cu_b, bs, out)
    e_ev.record()
    torch.cuda.synchronize()
    hash_us = s_ev.elapsed_time(e_ev) * 1e3 / reps
    hs = out.cpu().numpy().view(np.uint32)
    per_seq = [hs[cu_b_h[i]:cu_b_h[i + 1]] for i in range(len(seqs))]

    # the library's own time: inputs already packed as int32 / uint32 arrays
    import ctypes
    lib = pa.load_library()
    toks32 = toks.astype(np.int32)
    cu_tok = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    nblk = -(-lens // bs)
    offs = np.concatenate([[0], np.cumsum(nblk)]).astype(np.int64)
    tables_out = np.zeros(int(nblk.sum()), dtype=np.int32)
    hs32 = np.ascontiguousarray(hs, dtype=np.uint32)
    pool = int(lens.sum() // bs + len(seqs) + 64)

    def per_request(with_hashes):
        bm = pa.BlockManager(pool, bs)
        tp, hp, op = toks32.ctypes.data, hs32.ctypes.data, tables_out.ctypes.data
        t0 = time.perf_counter()
        for i in range(len(seqs)):
            st = lib.pa_bm_allocate(bm.h, tp + 4 * int(cu_tok[i]), int(lens[i]),
                                    hp + 4 * int(cu_b_h[i]) if with_hashes else None,
                                    op + 4 * int(offs[i]))
            assert st == 0
        dt = time.perf_counter() - t0
        used = bm.num_used()
        bm.close()
        return dt, used

    def one_call():
        bm = pa.BlockManager(pool, bs)
        done = ctypes.c_int32(0)
        t0 = time.perf_counter()
        st = lib.pa_bm_allocate_batch(bm.h, toks32.ctypes.data, cu_tok.ctypes.data, len(seqs),
                                      hs32.ctypes.data, cu_b_h.ctypes.data, tables_out.ctypes.data,
                                      ctypes.byref(done))
        dt = time.perf_counter() - t0
        assert st == 0 and done.value == len(seqs)
        used = bm.num_used()
        bm.close()
        return dt, used

    def through_binding():
        bm = pa.BlockManager(pool, bs)
        t0 = time.perf_counter()
        for x, h in zip(seqs, per_seq):
            bm.allocate(x, block_hashes=h)
        dt = time.perf_counter() - t0
        bm.close()
        return dt

    t_given, used = min(per_request(True) for _ in range(3))
    t_host, _ = min(per_request(False) for _ in range(3))
    t_batch, used_b = min(one_call() for _ in range(3))
    assert used_b == used
    t_py = through_binding()
    return {"requests": len(seqs), "tokens": int(lens.sum()), "block_size": bs,
            "gpu_hash_us": round(hash_us, 2), "gpu_hash_Mtokens_per_s": round(lens.sum() / hash_us, 1),
            "host_alloc_ms_hashes_given": round(t_given * 1e3, 3),
            "host_alloc_ms_hashing_on_host": round(t_host * 1e3, 3),
            "host_alloc_ms_one_batch_call": round(t_batch * 1e3, 3),
            "host_alloc_ms_python_lists_through_binding": round(t_py * 1e3, 2),
            "blocks_used": used,
            "note": "library times: packed arrays, one C call per request or one call for the "
                    "batch (best of 3); the binding time includes converting Python token lists"}


def run_reference(args, cfg, world):
    """Reference arm: the CPU oracle as it stands, on the host cores. Each step is a
    bounded sample of the workload: the oracle's decode of 2 of its sequences, on
    pools the oracle built itself (setup rows and the new tokens already stored)."""
    w = generate(cfg)
    pools = oracle_pools_for(w)
    per_step = 2
    times, byts = [], []
    for i in range(args.warmup + args.steps):
        dt, nb = 0.0, 0
        for j in range(per_step):
            a, b = oracle_decode_one(w, pools, (i * per_step + j) % w.num_seqs)
            dt += a
            nb += b
        if i >= args.warmup:
            times.append(dt)
            byts.append(nb)
    tot = sum(times)
    value = sum(byts) / tot / 1e9
    cores, blas = host_threads()
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot / len(times), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": cfg.name, "sample_per_step": f"{per_step} of {w.num_seqs} sequences"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "blas_threads": blas, "kind": "oracle",
                             "sample": f"oracle decode of {per_step} sequences per step"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
