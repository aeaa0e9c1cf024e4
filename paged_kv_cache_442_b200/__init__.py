"""Python binding of libpa.so, the B200 paged KV-cache library.

Argument marshalling only: every function here checks tensor dtypes/devices,
turns torch tensors into device pointers and calls the C entry point of the same
name (declared in include/pa.h). All arithmetic runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback. If libpa.so is missing or cannot be
loaded, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libpa.so")

PA_OK = 0
STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_BAD_INDEX",
                4: "PA_ERR_CUDA", 5: "PA_ERR_TIMEOUT", 6: "PA_ERR_NO_BLOCKS"}

# every extern "C" function include/pa.h declares
EXPORTED = ("pa_bm_create", "pa_bm_destroy", "pa_bm_allocate", "pa_bm_allocate_batch", "pa_bm_free",
            "pa_bm_append",
            "pa_bm_num_used", "pa_bm_ref_counts", "pa_block_hashes",
            "pa_store_kvcache", "pa_copy_blocks", "pa_decode_default_partition", "pa_decode_workspace_size",
            "pa_decode", "pa_store_decode", "pa_decode_shared_prefix",
            "pa_decode_shared_prefix_workspace_size", "pa_decode_no_alloc", "pa_prefill", "pa_store_prefill",
            "pa_store_kvcache_fp8", "pa_decode_fp8", "pa_set_debug_checks", "pa_set_wait_limit_ns",
            "pa_check_device_errors", "pa_status_string", "pa_version")

# size of the library-owned scratch of pa_decode_no_alloc (include/pa.h)
DECODE_NO_ALLOC_SCRATCH_BYTES = 8 * 1024 * 1024


class PAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


class pa_cache_desc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


_lib = None


def load_library(path: str | None = None):
    """Load libpa.so (once). Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} not found: build it with `python -m paged_kv_cache_442_b200.build`"
                          " (the CUDA library is required; there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.pa_store_kvcache.argtypes = [vp, vp, vp, vp, pa_cache_desc, vp, i32, vp]
    lib.pa_store_kvcache.restype = ctypes.c_int
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.pa_bm_create.argtypes = [i32, i32, vp]
    lib.pa_bm_create.restype = vp
    lib.pa_bm_destroy.argtypes = [vp]
    lib.pa_bm_destroy.restype = None
    lib.pa_bm_allocate.argtypes = [vp, vp, i32, vp, vp]
    lib.pa_bm_allocate.restype = ctypes.c_int
    lib.pa_bm_allocate_batch.argtypes = [vp, vp, vp, i32, vp, vp, vp, i32p]
    lib.pa_bm_allocate_batch.restype = ctypes.c_int
    lib.pa_bm_free.argtypes = [vp, vp, i32]
    lib.pa_bm_free.restype = ctypes.c_int
    lib.pa_bm_append.argtypes = [vp, vp, i32p, i32, i32, i32, i32p, i32p, i32p]
    lib.pa_bm_append.restype = ctypes.c_int
    lib.pa_bm_num_used.argtypes = [vp]
    lib.pa_bm_num_used.restype = i32
    lib.pa_bm_ref_counts.argtypes = [vp, vp]
    lib.pa_bm_ref_counts.restype = ctypes.c_int
    lib.pa_block_hashes.argtypes = [vp, vp, vp, i32, i32, vp, vp]
    lib.pa_block_hashes.restype = ctypes.c_int
    lib.pa_copy_blocks.argtypes = [vp, vp, pa_cache_desc, vp, vp, i32, vp]
    lib.pa_copy_blocks.restype = ctypes.c_int
    lib.pa_decode_default_partition.argtypes = [i32, i32, i32]
    lib.pa_decode_default_partition.restype = i32
    lib.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.pa_decode_workspace_size.restype = sz
    lib.pa_decode.argtypes = [vp, vp, vp, vp, pa_cache_desc, vp, i32, vp, i32, i32, ctypes.c_float,
                              i32, i32, vp, sz, vp]
    lib.pa_decode.restype = ctypes.c_int
    lib.pa_store_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, pa_cache_desc, vp, i32, vp, i32, i32,
                                    ctypes.c_float, i32, i32, vp, sz, vp]
    lib.pa_store_decode.restype = ctypes.c_int
    lib.pa_decode_shared_prefix.argtypes = [vp, vp, vp, vp, pa_cache_desc, vp, i32, vp, i32, i32,
                                            ctypes.c_float, i32, vp, i32, i32, vp, sz, vp]
    lib.pa_decode_shared_prefix.restype = ctypes.c_int
    lib.pa_decode_shared_prefix_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.pa_decode_shared_prefix_workspace_size.restype = sz
    lib.pa_decode_no_alloc.argtypes = [vp, vp, vp, vp, pa_cache_desc, vp, i32, vp, i32, i32,
                                       ctypes.c_float, i32, i32, vp]
    lib.pa_decode_no_alloc.restype = ctypes.c_int
    lib.pa_prefill.argtypes = [vp, vp, vp, vp, pa_cache_desc, vp, i32, vp, vp, i32, i32, i32, i32,
                               ctypes.c_float, vp]
    lib.pa_prefill.restype = ctypes.c_int
    lib.pa_store_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, pa_cache_desc, vp, i32, vp, vp, i32,
                                     i32, i32, i32, ctypes.c_float, vp]
    lib.pa_store_prefill.restype = ctypes.c_int
    lib.pa_store_kvcache_fp8.argtypes = [vp, vp, vp, vp, vp, vp, pa_cache_desc, vp, i32, vp]
    lib.pa_store_kvcache_fp8.restype = ctypes.c_int
    lib.pa_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, pa_cache_desc, vp, i32, vp, i32, i32,
                                  ctypes.c_float, i32, i32, vp, sz, vp]
    lib.pa_decode_fp8.restype = ctypes.c_int
    lib.pa_set_debug_checks.argtypes = [ctypes.c_int]
    lib.pa_set_debug_checks.restype = None
    lib.pa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.pa_set_wait_limit_ns.restype = None
    lib.pa_check_device_errors.argtypes = [vp]
    lib.pa_check_device_errors.restype = ctypes.c_int
    lib.pa_status_string.argtypes = [ctypes.c_int]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_version.restype = i32
    _lib = lib
    return lib


# ----------------------------------------------------------------- marshalling
def _torch():
    import torch
    return torch


def _check(t, name, dtype, ndim=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    return t


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(_torch().cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() else ctypes.c_void_p(0)


def _raise(fn, status):
    if status != PA_OK:
        raise PAError(fn, status)


def cache_desc(k_cache) -> pa_cache_desc:
    """Pool shape [num_blocks, block_size, num_kv_heads, head_dim] as the C struct."""
    nb, bs, hkv, d = k_cache.shape
    return pa_cache_desc(nb, bs, hkv, d)


# ----------------------------------------------------------------- entry points
def pa_store_kvcache(k, v, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """k_cache[slot_mapping[t]] = k[t], v_cache[...] = v[t] (slot -1 skips)."""
    torch = _torch()
    lib = load_library()
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(slot_mapping, "slot_mapping", torch.int32, 1)
    if k.shape != v.shape or k_cache.shape != v_cache.shape:
        raise ValueError("k/v and k_cache/v_cache shapes must match")
    if k.shape[0] != slot_mapping.shape[0] or tuple(k.shape[1:]) != tuple(k_cache.shape[2:]):
        raise ValueError("k must be [num_tokens, num_kv_heads, head_dim] matching the pool")
    st = lib.pa_store_kvcache(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache),
                              _ptr(slot_mapping), int(k.shape[0]), _stream(stream))
    _raise("pa_store_kvcache", st)


def pa_decode_default_partition(num_seqs: int, num_kv_heads: int, max_context_len: int) -> int:
    return int(load_library().pa_decode_default_partition(num_seqs, num_kv_heads, max_context_len))


def pa_decode_workspace_size(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int,
                             partition_size: int) -> int:
    return int(load_library().pa_decode_workspace_size(num_seqs, num_q_heads, head_dim,
                                                       max_context_len, partition_size))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
              max_context_len: int, partition_size: int = 0, workspace=None, stream=None) -> None:
    """Paged decode attention into `out` [num_seqs, Hq, D] (bf16)."""
    torch = _torch()
    lib = load_library()
    _check(out, "out", torch.bfloat16, 3)
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(context_lens, "context_lens", torch.int32, 1)
    B, Hq, D = q.shape
    if tuple(out.shape) != (B, Hq, D) or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("out/q/block_tables/context_lens disagree on num_seqs")
    ws_bytes = 0
    if workspace is not None:
        _check(workspace, "workspace", workspace.dtype)
        ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache),
                       _ptr(block_tables), int(block_tables.shape[1]), _ptr(context_lens), int(B),
                       int(Hq), float(scale), int(max_context_len), int(partition_size),
                       _ptr(workspace) if workspace is not None else ctypes.c_void_p(0), ws_bytes,
                       _stream(stream))
    _raise("pa_decode", st)


def _check_fp8_pools(torch, k_codes, v_codes, k_scales, v_scales):
    _check(k_codes, "k_codes", torch.uint8, 4)
    _check(v_codes, "v_codes", torch.uint8, 4)
    _check(k_scales, "k_scales", torch.float32, 2)
    _check(v_scales, "v_scales", torch.float32, 2)
    nb, bs, hkv, _ = k_codes.shape
    if k_codes.shape != v_codes.shape or k_scales.shape != v_scales.shape:
        raise ValueError("K and V pools must have the same shapes")
    if tuple(k_scales.shape) != (hkv, nb * bs):
        raise ValueError("scales must be [num_kv_heads, num_blocks * block_size] fp32")


def pa_store_kvcache_fp8(k, v, k_codes, v_codes, k_scales, v_scales, slot_mapping,
                         stream=None) -> None:
    """Quantise k[t], v[t] (bf16) into the e4m3 pools at row slot_mapping[t]: codes
    uint8 [num_blocks, bs, Hkv, D], per-row scales fp32 [Hkv, num_blocks * bs]."""
    torch = _torch()
    lib = load_library()
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    _check_fp8_pools(torch, k_codes, v_codes, k_scales, v_scales)
    _check(slot_mapping, "slot_mapping", torch.int32, 1)
    if k.shape != v.shape or k.shape[0] != slot_mapping.shape[0] or \
            tuple(k.shape[1:]) != tuple(k_codes.shape[2:]):
        raise ValueError("k must be [num_tokens, num_kv_heads, head_dim] matching the pool")
    st = lib.pa_store_kvcache_fp8(_ptr(k), _ptr(v), _ptr(k_codes), _ptr(v_codes), _ptr(k_scales),
                                  _ptr(v_scales), cache_desc(k_codes), _ptr(slot_mapping),
                                  int(k.shape[0]), _stream(stream))
    _raise("pa_store_kvcache_fp8", st)


def pa_decode_fp8(out, q, k_codes, v_codes, k_scales, v_scales, block_tables, context_lens,
                  scale: float, max_context_len: int, partition_size: int = 0, workspace=None,
                  stream=None) -> None:
    """Paged decode attention over e4m3 pools into `out` [num_seqs, Hq, D] (bf16)."""
    torch = _torch()
    lib = load_library()
    _check(out, "out", torch.bfloat16, 3)
    _check(q, "q", torch.bfloat16, 3)
    _check_fp8_pools(torch, k_codes, v_codes, k_scales, v_scales)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(context_lens, "context_lens", torch.int32, 1)
    B, Hq, D = q.shape
    if tuple(out.shape) != (B, Hq, D) or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("out/q/block_tables/context_lens disagree on num_seqs")
    ws_bytes = 0
    if workspace is not None:
        _check(workspace, "workspace", workspace.dtype)
        ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.pa_decode_fp8(_ptr(out), _ptr(q), _ptr(k_codes), _ptr(v_codes), _ptr(k_scales),
                           _ptr(v_scales), cache_desc(k_codes), _ptr(block_tables),
                           int(block_tables.shape[1]), _ptr(context_lens), int(B), int(Hq),
                           float(scale), int(max_context_len), int(partition_size),
                           _ptr(workspace) if workspace is not None else ctypes.c_void_p(0),
                           ws_bytes, _stream(stream))
    _raise("pa_decode_fp8", st)


class BlockManager:
    """The library's host block manager (include/pa.h, pa_bm_*): block tables with
    hash-chained prefix sharing, reference counts, and decode append with
    copy-on-write. Host memory only; not thread-safe."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        import numpy as np
        self._np = np
        self.lib = load_library()
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
        self.h = self.lib.pa_bm_create(self.num_blocks, self.block_size,
                                       order.ctypes.data if order is not None else None)
        if not self.h:
            raise ValueError("bad sizes or free_order is not a permutation of the pool")
        self._order = order

    def close(self):
        if self.h:
            self.lib.pa_bm_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate(self, token_ids, block_hashes=None) -> list:
        np = self._np
        toks = np.ascontiguousarray(token_ids, dtype=np.int32)
        table = np.zeros(-(-len(toks) // self.block_size), dtype=np.int32)
        hs = None if block_hashes is None else np.ascontiguousarray(block_hashes, dtype=np.uint32)
        st = self.lib.pa_bm_allocate(self.h, toks.ctypes.data, len(toks),
                                     hs.ctypes.data if hs is not None else None, table.ctypes.data)
        _raise("pa_bm_allocate", st)
        return table.tolist()

    def allocate_batch(self, requests, block_hashes=None):
        """Tables of several requests in one library call, in order. Returns (tables,
        number allocated); when the pool runs out the status is raised after the
        allocated prefix is recorded in the exception's `done` attribute."""
        np = self._np
        lens = np.array([len(r) for r in requests], dtype=np.int64)
        cu = np.zeros(len(requests) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(lens)
        toks = (np.concatenate([np.asarray(r, dtype=np.int32) for r in requests])
                if len(requests) and cu[-1] else np.zeros(1, dtype=np.int32))
        nblk = -(-lens // self.block_size)
        out = np.zeros(max(1, int(nblk.sum())), dtype=np.int32)
        hs = cub = None
        if block_hashes is not None:
            hs = np.concatenate([np.asarray(h, dtype=np.uint32) for h in block_hashes]
                                + [np.zeros(1, np.uint32)])
            cub = np.zeros(len(requests) + 1, dtype=np.int32)
            cub[1:] = np.cumsum([len(h) for h in block_hashes])
        done = ctypes.c_int32(0)
        st = self.lib.pa_bm_allocate_batch(self.h, toks.ctypes.data, cu.ctypes.data, len(requests),
                                           hs.ctypes.data if hs is not None else None,
                                           cub.ctypes.data if cub is not None else None,
                                           out.ctypes.data, ctypes.byref(done))
        offs = np.concatenate([[0], np.cumsum(nblk)])
        tables = [out[offs[i]:offs[i + 1]].tolist() for i in range(done.value)]
        if st != PA_OK:
            err = PAError("pa_bm_allocate_batch", st)
            err.done = done.value
            err.tables = tables
            raise err
        return tables

    def free(self, table) -> None:
        t = self._np.ascontiguousarray(table, dtype=self._np.int32)
        _raise("pa_bm_free", self.lib.pa_bm_free(self.h, t.ctypes.data, len(t)))

    def append(self, table: list, pos: int, token_id: int):
        """Slot of position pos; `table` (a list) is updated in place. Returns
        (slot, (src, dst) copy or None)."""
        np = self._np
        buf = np.zeros(len(table) + 1, dtype=np.int32)
        buf[:len(table)] = table
        n = ctypes.c_int32(len(table))
        slot, src, dst = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
        st = self.lib.pa_bm_append(self.h, buf.ctypes.data, ctypes.byref(n), len(buf), int(pos),
                                   int(token_id), ctypes.byref(slot), ctypes.byref(src),
                                   ctypes.byref(dst))
        _raise("pa_bm_append", st)
        table[:] = buf[:n.value].tolist()
        return slot.value, (None if src.value < 0 else (src.value, dst.value))

    def num_used(self) -> int:
        return int(self.lib.pa_bm_num_used(self.h))

    def ref_counts(self):
        out = self._np.zeros(self.num_blocks, dtype=self._np.int32)
        _raise("pa_bm_ref_counts", self.lib.pa_bm_ref_counts(self.h, out.ctypes.data))
        return out


def pa_block_hashes(token_ids, cu_tokens, cu_blocks, block_size: int, hashes_out, stream=None) -> None:
    """Chained hash of every full block of a batch of sequences (device tensors:
    int32 tokens back to back, int32 token and block offsets, uint32-sized output)."""
    torch = _torch()
    lib = load_library()
    _check(token_ids, "token_ids", torch.int32, 1)
    _check(cu_tokens, "cu_tokens", torch.int32, 1)
    _check(cu_blocks, "cu_blocks", torch.int32, 1)
    _check(hashes_out, "hashes_out", hashes_out.dtype, 1)
    if hashes_out.element_size() != 4 or cu_tokens.shape != cu_blocks.shape:
        raise ValueError("hashes_out must hold 32-bit values; cu_tokens and cu_blocks must match")
    st = lib.pa_block_hashes(_ptr(token_ids), _ptr(cu_tokens), _ptr(cu_blocks),
                             int(cu_tokens.shape[0]) - 1, int(block_size), _ptr(hashes_out),
                             _stream(stream))
    _raise("pa_block_hashes", st)


def pa_copy_blocks(k_cache, v_cache, src_blocks, dst_blocks, stream=None) -> None:
    """Copy-on-write: block dst_blocks[i] of both pools becomes a copy of block
    src_blocks[i] (destinations distinct, and not also sources)."""
    torch = _torch()
    lib = load_library()
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(src_blocks, "src_blocks", torch.int32, 1)
    _check(dst_blocks, "dst_blocks", torch.int32, 1)
    if src_blocks.shape != dst_blocks.shape or k_cache.shape != v_cache.shape:
        raise ValueError("src/dst lengths or the two pools' shapes disagree")
    st = lib.pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), cache_desc(k_cache), _ptr(src_blocks),
                            _ptr(dst_blocks), int(src_blocks.shape[0]), _stream(stream))
    _raise("pa_copy_blocks", st)


def pa_store_decode(new_k, new_v, slot_mapping, out, q, k_cache, v_cache, block_tables,
                    context_lens, scale: float, max_context_len: int, partition_size: int = 0,
                    workspace=None, stream=None) -> None:
    """Store each sequence's new K/V row at slot_mapping[s] (the slot of its last
    position, or -1), then decode: the same result as pa_store_kvcache followed by
    pa_decode, in one launch on the tensor-core path."""
    torch = _torch()
    lib = load_library()
    _check(new_k, "new_k", torch.bfloat16, 3)
    _check(new_v, "new_v", torch.bfloat16, 3)
    _check(slot_mapping, "slot_mapping", torch.int32, 1)
    _check(out, "out", torch.bfloat16, 3)
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(context_lens, "context_lens", torch.int32, 1)
    B, Hq, D = q.shape
    if tuple(out.shape) != (B, Hq, D) or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("out/q/block_tables/context_lens disagree on num_seqs")
    row = (B, k_cache.shape[2], k_cache.shape[3])
    if tuple(new_k.shape) != row or tuple(new_v.shape) != row or slot_mapping.shape[0] != B:
        raise ValueError("new_k/new_v must be [num_seqs, Hkv, D] and slot_mapping [num_seqs]")
    ws_bytes = 0
    if workspace is not None:
        _check(workspace, "workspace", workspace.dtype)
        ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.pa_store_decode(_ptr(new_k), _ptr(new_v), _ptr(slot_mapping), _ptr(out), _ptr(q),
                             _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache), _ptr(block_tables),
                             int(block_tables.shape[1]), _ptr(context_lens), int(B), int(Hq),
                             float(scale), int(max_context_len), int(partition_size),
                             _ptr(workspace) if workspace is not None else ctypes.c_void_p(0),
                             ws_bytes, _stream(stream))
    _raise("pa_store_decode", st)


def pa_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                            max_context_len: int, shared_blocks, shared_len: int,
                            partition_size: int = 0, workspace=None, stream=None) -> None:
    """Decode of a batch whose first shared_len positions live in the same blocks
    (shared_blocks, int32 device tensor) for every sequence: the shared prefix attended
    once for all of them, then the rest."""
    torch = _torch()
    lib = load_library()
    _check(out, "out", torch.bfloat16, 3)
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(context_lens, "context_lens", torch.int32, 1)
    _check(shared_blocks, "shared_blocks", torch.int32, 1)
    B, Hq, D = q.shape
    if tuple(out.shape) != (B, Hq, D) or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("out/q/block_tables/context_lens disagree on num_seqs")
    if shared_len and shared_blocks.shape[0] * k_cache.shape[1] < shared_len:
        raise ValueError("shared_blocks must cover shared_len positions")
    ws_bytes = 0
    if workspace is not None:
        _check(workspace, "workspace", workspace.dtype)
        ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.pa_decode_shared_prefix(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                     cache_desc(k_cache), _ptr(block_tables),
                                     int(block_tables.shape[1]), _ptr(context_lens), int(B), int(Hq),
                                     float(scale), int(max_context_len), _ptr(shared_blocks),
                                     int(shared_len), int(partition_size),
                                     _ptr(workspace) if workspace is not None else ctypes.c_void_p(0),
                                     ws_bytes, _stream(stream))
    _raise("pa_decode_shared_prefix", st)


def shared_prefix_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                            shared_len, partition_size=0, device="cuda"):
    """Allocate (with torch) the scratch pa_decode_shared_prefix needs; returns
    (workspace, partition size) as decode_workspace does."""
    torch = _torch()
    lib = load_library()
    rest = max(1, max_context_len - shared_len)
    P = partition_size or pa_decode_default_partition(num_seqs, num_kv_heads, rest)
    nbytes = int(lib.pa_decode_shared_prefix_workspace_size(num_seqs, num_q_heads, head_dim,
                                                            max_context_len, shared_len, P))
    return torch.empty(max(nbytes, 16) // 4, dtype=torch.float32, device=device), P


def pa_decode_no_alloc(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                       max_context_len: int, partition_size: int = 0, stream=None) -> None:
    """pa_decode for callers that cannot allocate device memory.

    Same result as pa_decode, but the split-K scratch is a fixed array the library
    owns (DECODE_NO_ALLOC_SCRATCH_BYTES per GPU), so the caller passes no
    workspace and nothing is allocated. Sizes that need more scratch than that are
    rejected; calls on one GPU share the array, so they must not overlap.
    """
    torch = _torch()
    lib = load_library()
    _check(out, "out", torch.bfloat16, 3)
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(context_lens, "context_lens", torch.int32, 1)
    B, Hq, D = q.shape
    if tuple(out.shape) != (B, Hq, D) or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("out/q/block_tables/context_lens disagree on num_seqs")
    st = lib.pa_decode_no_alloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                cache_desc(k_cache), _ptr(block_tables), int(block_tables.shape[1]),
                                _ptr(context_lens), int(B), int(Hq), float(scale),
                                int(max_context_len), int(partition_size), _stream(stream))
    if st == 2:
        P = partition_size or pa_decode_default_partition(B, k_cache.shape[2], max_context_len)
        need = pa_decode_workspace_size(B, Hq, D, max_context_len, P)
        if need > DECODE_NO_ALLOC_SCRATCH_BYTES:
            raise PAError(f"pa_decode_no_alloc (needs {need} bytes of split-K scratch, more than "
                          f"the library's fixed {DECODE_NO_ALLOC_SCRATCH_BYTES}; use a larger "
                          f"partition_size or pa_decode with a workspace)", st)
    _raise("pa_decode_no_alloc", st)


def pa_prefill(out, q, k_cache, v_cache, block_tables, cu_seqlens_q, context_lens, scale: float,
               max_q_len: int, stream=None) -> None:
    """Causal paged prefill into `out` [total_q, Hq, D] (bf16)."""
    torch = _torch()
    lib = load_library()
    _check(out, "out", torch.bfloat16, 3)
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _check(context_lens, "context_lens", torch.int32, 1)
    Tq, Hq, D = q.shape
    B = context_lens.shape[0]
    if tuple(out.shape) != (Tq, Hq, D) or cu_seqlens_q.shape[0] != B + 1 or block_tables.shape[0] != B:
        raise ValueError("out/q/cu_seqlens_q/block_tables/context_lens shapes disagree")
    st = lib.pa_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache),
                        _ptr(block_tables), int(block_tables.shape[1]), _ptr(cu_seqlens_q),
                        _ptr(context_lens), int(B), int(Hq), int(Tq), int(max_q_len), float(scale),
                        _stream(stream))
    _raise("pa_prefill", st)


def pa_store_prefill(new_k, new_v, slot_mapping, out, q, k_cache, v_cache, block_tables,
                     cu_seqlens_q, context_lens, scale: float, max_q_len: int,
                     stream=None) -> None:
    """Store the new tokens' K/V rows at slot_mapping (their block-table slots) and run
    the causal paged prefill in one launch: the same result, and pool, as
    pa_store_kvcache followed by pa_prefill."""
    torch = _torch()
    lib = load_library()
    _check(new_k, "new_k", torch.bfloat16, 3)
    _check(new_v, "new_v", torch.bfloat16, 3)
    _check(slot_mapping, "slot_mapping", torch.int32, 1)
    _check(out, "out", torch.bfloat16, 3)
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(block_tables, "block_tables", torch.int32, 2)
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _check(context_lens, "context_lens", torch.int32, 1)
    Tq, Hq, D = q.shape
    B = context_lens.shape[0]
    if tuple(out.shape) != (Tq, Hq, D) or cu_seqlens_q.shape[0] != B + 1 or block_tables.shape[0] != B:
        raise ValueError("out/q/cu_seqlens_q/block_tables/context_lens shapes disagree")
    row = (Tq, k_cache.shape[2], k_cache.shape[3])
    if tuple(new_k.shape) != row or tuple(new_v.shape) != row or slot_mapping.shape[0] != Tq:
        raise ValueError("new_k/new_v must be [total_q, Hkv, D] and slot_mapping [total_q]")
    st = lib.pa_store_prefill(_ptr(new_k), _ptr(new_v), _ptr(slot_mapping), _ptr(out), _ptr(q),
                              _ptr(k_cache), _ptr(v_cache), cache_desc(k_cache), _ptr(block_tables),
                              int(block_tables.shape[1]), _ptr(cu_seqlens_q), _ptr(context_lens),
                              int(B), int(Hq), int(Tq), int(max_q_len), float(scale), _stream(stream))
    _raise("pa_store_prefill", st)


def pa_set_debug_checks(on: bool) -> None:
    load_library().pa_set_debug_checks(1 if on else 0)


def pa_set_wait_limit_ns(ns: int) -> None:
    """Test hook: bound of the waits between the tensor-core kernels' roles (0 = the
    default 2 s). See include/pa.h."""
    load_library().pa_set_wait_limit_ns(int(ns))


def pa_check_device_errors(stream=None) -> int:
    """Synchronise, read and clear the device error word; returns a status code."""
    return int(load_library().pa_check_device_errors(_stream(stream)))


def pa_status_string(status: int) -> str:
    return load_library().pa_status_string(int(status)).decode()


def pa_version() -> int:
    return int(load_library().pa_version())


def decode_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                     partition_size=0, device="cuda"):
    """Allocate (with torch) the scratch pa_decode needs.

    Returns (workspace tensor or None, partition size); pass both to pa_decode so
    the split it runs is the one the scratch was sized for.
    """
    torch = _torch()
    P = partition_size or pa_decode_default_partition(num_seqs, num_kv_heads, max_context_len)
    nbytes = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len, P)
    if nbytes == 0:
        return None, P
    return torch.empty(nbytes // 4, dtype=torch.float32, device=device), P
