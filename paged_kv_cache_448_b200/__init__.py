"""libpaged: paged KV-cache decode attention for B200 (sm_100a) — Python binding.

Every op here marshals arguments into one call of the C ABI in
``include/paged.h`` (``libpaged.so``, built in-tree); all compute runs in the
library's CUDA kernels. PyTorch supplies device memory and the current stream
only. If the library is missing the first op raises ``ImportError``.

Ops:
  * ``reshape_and_cache`` — scatter a step's new K/V rows into cache slots.
  * ``decode`` — paged attention of one query token per sequence.
  * ``BlockAllocator``, ``build_block_table``, ``build_slot_mapping`` — host
    allocator and integer-table builders (no GPU).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _native
from ._native import PagedError, check

__all__ = ["reshape_and_cache", "decode", "decode_noalloc", "decode_noalloc_check",
           "inject_wait_timeout", "decode_workspace",
           "decode_workspace_size",
           "decode_partition_tokens", "decode_check", "chunked_prefill",
           "chunked_prefill_workspace", "chunked_prefill_workspace_size", "copy_blocks", "sha256", "block_hash",
           "prompt_block_hashes", "BlockAllocator",
           "build_block_table",
           "build_slot_mapping", "PagedError", "dtype_code"]


def dtype_code(t) -> int:
    """pa_dtype of a torch tensor (uint8 / float8_e4m3fn storage is E4M3)."""
    import torch
    if t.dtype == torch.float16:
        return _native.PA_F16
    if t.dtype == torch.bfloat16:
        return _native.PA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return _native.PA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_handle(stream) -> int | None:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, *, k_scale=None,
                      v_scale=None, stream=None) -> None:
    """key/value [T, Hkv, D] f16|bf16; caches [NB, BS, Hkv, D] (same dtype, or uint8 E4M3
    with fp32 k_scale/v_scale [Hkv]); slot_mapping int32 [T] (negative = skip)."""
    T, Hkv, D = key.shape
    NB, BS = key_cache.shape[:2]
    check(_native.lib().pa_reshape_and_cache(
        _ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache), _ptr(slot_mapping), T, Hkv,
        D, BS, NB, dtype_code(key), dtype_code(key_cache), _ptr(k_scale), _ptr(v_scale),
        _stream_handle(stream)))


def decode_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_context_len, partition_tokens=0,
                            cache_dtype: int = _native.PA_F16) -> int:
    """Partition length pa_decode uses (>= max_context_len: one pass);
    cache_dtype is a pa_dtype code."""
    return int(_native.lib().pa_decode_partition_tokens(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
        partition_tokens, int(cache_dtype)))


def decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                          max_context_len, partition_tokens=0,
                          cache_dtype: int = _native.PA_F16) -> int:
    return int(_native.lib().pa_decode_workspace_size(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
        partition_tokens, int(cache_dtype)))


def decode_workspace(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                     partition_tokens=0, device="cuda", stream=None,
                     cache_dtype: int = _native.PA_F16):
    """A device workspace (torch uint8) of the size pa_decode needs, error word zeroed."""
    import torch
    n = decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                              max_context_len, partition_tokens, cache_dtype)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    check(_native.lib().pa_workspace_init(_ptr(ws), ws.numel(), _stream_handle(stream)))
    return ws


def decode(out, query, key_cache, value_cache, block_tables, context_lens, max_context_len: int,
           scale: float, *, k_scale=None, v_scale=None, partition_tokens: int = 0,
           workspace=None, stream=None):
    """out/query [S, H, D] f16|bf16; caches [NB, BS, Hkv, D]; block_tables int32
    [S, max_blocks]; context_lens int32 [S]; max_context_len >= every context length.
    Returns ``out``."""
    S, H, D = query.shape
    NB, BS, Hkv = key_cache.shape[:3]
    if workspace is None:
        workspace = decode_workspace(S, H, Hkv, D, BS, max_context_len, partition_tokens,
                                     device=query.device, stream=stream,
                                     cache_dtype=dtype_code(key_cache))
    check(_native.lib().pa_decode(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, H, Hkv, D, BS, NB,
        float(scale), dtype_code(query), dtype_code(key_cache), _ptr(k_scale), _ptr(v_scale),
        int(partition_tokens), _ptr(workspace), workspace.numel(), _stream_handle(stream)))
    return out


def decode_noalloc(out, query, key_cache, value_cache, block_tables, context_lens,
                   max_context_len: int, scale: float, *, k_scale=None, v_scale=None,
                   partition_tokens: int = 0, stream=None):
    """decode() for callers that cannot allocate device memory: the library's
    own static 32 MiB device scratch replaces the workspace (pa_decode_noalloc).
    Calls that overlap on the GPU race on that scratch. Returns ``out``."""
    S, H, D = query.shape
    NB, BS, Hkv = key_cache.shape[:3]
    check(_native.lib().pa_decode_noalloc(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, H, Hkv, D, BS, NB,
        float(scale), dtype_code(query), dtype_code(key_cache), _ptr(k_scale), _ptr(v_scale),
        int(partition_tokens), _stream_handle(stream)))
    return out


def decode_check(workspace, stream=None) -> None:
    """Synchronise and raise PagedError if a decode on `workspace` met a bad
    table entry (PA_ERR_BAD_TABLE) or a pipeline wait gave up (PA_ERR_CUDA)."""
    check(_native.lib().pa_decode_check(_ptr(workspace), _stream_handle(stream)))


def decode_noalloc_check(stream=None) -> None:
    """decode_check for decode_noalloc: reads and clears the error word of the
    library's static scratch on the current device (pa_decode_noalloc_check)."""
    check(_native.lib().pa_decode_noalloc_check(_stream_handle(stream)))


def inject_wait_timeout(tile: int, wait_limit_ns: int) -> None:
    """Failure-detection test hook (pa_inject_wait_timeout): the next decode,
    decode_noalloc or chunked_prefill on this thread leaves out the loads of
    16-token tile `tile` of its first work unit and bounds every wait by
    `wait_limit_ns`; the wait for that tile runs out and the check call
    reports it. tile < 0 cancels."""
    check(_native.lib().pa_inject_wait_timeout(int(tile), int(wait_limit_ns)))


# ---------------------------------------------------------------- host side

def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def chunked_prefill_workspace_size(num_seqs, num_tokens, num_heads, num_kv_heads, head_dim,
                                   max_query_len, max_context_len,
                                   cache_dtype: int = _native.PA_F16) -> int:
    """Bytes pa_chunked_prefill needs; cache_dtype is a pa_dtype code (an
    E4M3 cache always takes the mma.sync kernel, which may split)."""
    return int(_native.lib().pa_chunked_prefill_workspace_size(
        num_seqs, num_tokens, num_heads, num_kv_heads, head_dim, max_query_len, max_context_len,
        int(cache_dtype)))


def chunked_prefill_workspace(num_seqs, num_tokens, num_heads, num_kv_heads, head_dim,
                              max_query_len, max_context_len, cache_dtype: int = _native.PA_F16,
                              device="cuda", stream=None):
    """A device workspace for pa_chunked_prefill, error word zeroed."""
    import torch
    n = chunked_prefill_workspace_size(num_seqs, num_tokens, num_heads, num_kv_heads, head_dim,
                                       max_query_len, max_context_len, cache_dtype)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    check(_native.lib().pa_workspace_init(_ptr(ws), ws.numel(), _stream_handle(stream)))
    return ws


def chunked_prefill(out, query, cu_query_lens, max_query_len: int, key_cache, value_cache,
                    block_tables, context_lens, max_context_len: int, scale: float, *,
                    k_scale=None, v_scale=None, workspace=None, stream=None):
    """Several query tokens per sequence (its last positions), causal
    (pa_chunked_prefill). out/query [T, H, D] f16|bf16; caches of the query's
    dtype, or E4M3 (uint8 / float8_e4m3fn) with k_scale / v_scale float32
    [Hkv]; cu_query_lens int32 [S+1]; context_lens include the query tokens."""
    T, H, D = query.shape
    NB, BS, Hkv = key_cache.shape[:3]
    S = context_lens.shape[0]
    if workspace is None:
        workspace = chunked_prefill_workspace(S, T, H, Hkv, D, max_query_len, max_context_len,
                                              dtype_code(key_cache), device=query.device,
                                              stream=stream)
    check(_native.lib().pa_chunked_prefill(
        _ptr(out), _ptr(query), _ptr(cu_query_lens), T, int(max_query_len), _ptr(key_cache),
        _ptr(value_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
        int(max_context_len), S, H, Hkv, D, BS, NB, float(scale), dtype_code(query),
        dtype_code(key_cache), _ptr(k_scale), _ptr(v_scale), _ptr(workspace), workspace.numel(),
        _stream_handle(stream)))
    return out


def copy_blocks(src_key_cache, src_value_cache, dst_key_cache, dst_value_cache, block_pairs, *,
                error_word=None, stream=None):
    """Copy whole blocks src[pairs[i, 0]] -> dst[pairs[i, 1]] (pa_copy_blocks).

    Caches are [num_blocks, ...] tensors on the GPU or in pinned host memory
    (value caches may both be None); block_pairs is an int32 [n, 2] tensor on
    the GPU or pinned. A block is one row along axis 0 of each cache.
    """
    n = int(block_pairs.shape[0]) if block_pairs.dim() == 2 else 0
    if block_pairs.dim() != 2 or block_pairs.shape[1] != 2 or not block_pairs.is_contiguous():
        raise ValueError("block_pairs must be a contiguous int32 [n, 2] tensor")
    bb = src_key_cache[0].numel() * src_key_cache.element_size()
    if dst_key_cache[0].numel() * dst_key_cache.element_size() != bb:
        raise ValueError("source and destination blocks differ in size")
    if src_value_cache is not None and (
            src_value_cache[0].numel() * src_value_cache.element_size() != bb or
            dst_value_cache[0].numel() * dst_value_cache.element_size() != bb):
        raise ValueError("value blocks differ in size from key blocks")
    check(_native.lib().pa_copy_blocks(
        _ptr(src_key_cache), _ptr(src_value_cache), _ptr(dst_key_cache), _ptr(dst_value_cache),
        _ptr(block_pairs), n, bb, src_key_cache.shape[0], dst_key_cache.shape[0],
        _ptr(error_word), _stream_handle(stream)))


def sha256(data: bytes) -> bytes:
    """SHA-256 of a byte string (pa_sha256)."""
    buf = ctypes.create_string_buffer(bytes(data), max(len(data), 1))
    out = ctypes.create_string_buffer(32)
    check(_native.lib().pa_sha256(buf, len(data), out))
    return out.raw


def block_hash(parent, tokens) -> bytes:
    """Hash of one block chained to its parent's (None for a prompt's first)."""
    t = _i32(tokens)
    par = None if parent is None else ctypes.create_string_buffer(bytes(parent), 32)
    out = ctypes.create_string_buffer(32)
    check(_native.lib().pa_block_hash(par, t.ctypes.data if t.size else None, t.size, out))
    return out.raw


def prompt_block_hashes(tokens, block_size: int) -> np.ndarray:
    """uint8 [len(tokens) // block_size, 32]: chained hashes of the full blocks."""
    t = _i32(tokens)
    n = t.size // block_size
    out = np.empty((max(n, 1), 32), np.uint8)
    check(_native.lib().pa_prompt_block_hashes(t.ctypes.data if t.size else None, t.size,
                                               block_size, out.ctypes.data))
    return out[:n]


class BlockAllocator:
    """Host free list with refcounts (pa_alloc_*)."""

    def __init__(self, num_blocks: int, initial_free_order=None):
        self._lib = _native.lib()
        order = None if initial_free_order is None else _i32(initial_free_order)
        h = ctypes.c_void_p()
        check(self._lib.pa_alloc_create(num_blocks, None if order is None else order.ctypes.data,
                                        ctypes.byref(h)))
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            self._lib.pa_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def allocate(self, n: int) -> list:
        ids = np.empty(max(n, 1), np.int32)
        check(self._lib.pa_alloc_allocate(self._h, n, ids.ctypes.data))
        return [int(i) for i in ids[:n]]

    def share(self, block_id: int) -> None:
        check(self._lib.pa_alloc_share(self._h, int(block_id)))

    def free(self, ids) -> None:
        a = _i32(ids)
        check(self._lib.pa_alloc_free(self._h, a.ctypes.data if a.size else None, a.size))

    def copy_on_write(self, block_id: int):
        """(block to write, must_copy): a shared block is replaced by a fresh one
        that the caller fills with copy_blocks (pa_alloc_copy_on_write)."""
        out, copy = ctypes.c_int32(), ctypes.c_int32()
        check(self._lib.pa_alloc_copy_on_write(self._h, int(block_id), ctypes.byref(out),
                                               ctypes.byref(copy)))
        return int(out.value), bool(copy.value)

    def acquire_prefix(self, hashes):
        """Blocks for a prompt's full-block hashes ([n, 32] uint8): cached ones
        are shared, the rest allocated and registered. Returns (ids, hits)."""
        h = np.ascontiguousarray(hashes, dtype=np.uint8).reshape(-1, 32)
        ids = np.empty(max(len(h), 1), np.int32)
        hits = ctypes.c_int32()
        check(self._lib.pa_alloc_acquire_prefix(self._h, h.ctypes.data if len(h) else None,
                                                len(h), ids.ctypes.data, ctypes.byref(hits)))
        return [int(i) for i in ids[:len(h)]], int(hits.value)

    def register_hash(self, block_id: int, h) -> None:
        b = np.ascontiguousarray(np.frombuffer(bytes(h), np.uint8))
        check(self._lib.pa_alloc_register_hash(self._h, int(block_id), b.ctypes.data))

    def lookup(self, h) -> int:
        b = np.ascontiguousarray(np.frombuffer(bytes(h), np.uint8))
        return int(self._lib.pa_alloc_lookup(self._h, b.ctypes.data))

    @property
    def num_free(self) -> int:
        return int(self._lib.pa_alloc_num_free(self._h))

    @property
    def num_blocks(self) -> int:
        return int(self._lib.pa_alloc_num_blocks(self._h))

    def refcount(self, block_id: int) -> int:
        return int(self._lib.pa_alloc_refcount(self._h, int(block_id)))

    def free_list(self) -> list:
        n = self.num_free
        out = np.empty(max(n, 1), np.int32)
        self._lib.pa_alloc_free_list(self._h, out.ctypes.data, n)
        return [int(i) for i in out[:n]]


def build_block_table(seq_block_ids, max_blocks_per_seq: int) -> np.ndarray:
    """int32 [S, max_blocks_per_seq] from per-sequence id lists; unused = -1."""
    rows = [_i32(ids) for ids in seq_block_ids]
    S = len(rows)
    ptrs = (ctypes.c_void_p * max(S, 1))(*[r.ctypes.data if r.size else None for r in rows])
    counts = _i32([r.size for r in rows]) if S else np.zeros(1, np.int32)
    out = np.empty((max(S, 1), max_blocks_per_seq), np.int32)
    check(_native.lib().pa_build_block_table(ctypes.cast(ptrs, ctypes.c_void_p),
                                             counts.ctypes.data, S, max_blocks_per_seq,
                                             out.ctypes.data))
    return out[:S]


def build_slot_mapping(block_tables, positions, block_size: int, seq_ids=None) -> np.ndarray:
    """int32 slots for (sequence, position) pairs; position < 0 gives -1."""
    bt = _i32(block_tables)
    pos = _i32(positions)
    sid = None if seq_ids is None else _i32(seq_ids)
    out = np.empty(max(pos.size, 1), np.int32)
    check(_native.lib().pa_build_slot_mapping(bt.ctypes.data, bt.shape[0], bt.shape[1],
                                              None if sid is None else sid.ctypes.data,
                                              pos.ctypes.data, pos.size, block_size,
                                              out.ctypes.data))
    return out[:pos.size]
