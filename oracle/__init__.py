"""CPU fp64 oracle for paged decode attention and reshape_and_cache.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline may import this package; the product path (``paged_kv_cache_448_b200``)
never does. The arithmetic lives in ``oracle.c`` (plain C, fp64, no blocking or
fusion); this module only compiles it with gcc on first use and marshals numpy
arrays. It shares no code with the CUDA library.

Functions mirror the pages' problem statement:

* ``decode`` — [P2] "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" §2.3
  (attention over the blocks a block table names) with the logical->physical
  translation of [P1] "vLLM框架中的KV cache优化与PagedAttention机制详解" §5.1.
* ``reshape_and_cache`` — writes rows into the cache layout of [P2] §2.2.
* ``chunked_prefill`` — the same attention for several query tokens per
  sequence (its last positions), each seeing itself and earlier tokens.
* ``slot_mapping`` — the address translation of [P3] "Paged KVCache：大模型推理
  显存管理优化方案" §2.3, page size counted in tokens.
* ``BlockManager`` (``oracle.block_manager``) — the free list of [P2] §2.2 with
  the reference counts of [P4] "大模型推理KV Cache内存管理与PagedAttention分页显存实战",
  and copy-on-write of a shared block before a write.
* ``copy_blocks`` — whole-block copies between or within caches: the private
  copy of a shared block ([P4]'s reference-counted sharing) and the migration
  of blocks between GPU memory and host memory ([P3] §5, Hybrid Cache; [P4]'s
  ``swap_space``).

Parity status: every function here is pinned by the ``-m "not gpu"`` tests
(format decoders exhaustively against numpy/torch, the E4M3 encoder against a
brute-force nearest search, decode against fp64
``torch.nn.functional.scaled_dot_product_attention`` on contiguous K/V, closed
forms and invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liborc.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODES = {"f16": 0, "bf16": 1, "e4m3": 2}
_ELEM_BYTES = {"f16": 2, "bf16": 2, "e4m3": 1}


def build(force: bool = False) -> str:
    """Compile oracle.c into liborc.so next to it (gcc, -O2, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-fPIC", "-shared",
             _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f32, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        lib.orc_decode_f16.argtypes = [ctypes.c_uint16]; lib.orc_decode_f16.restype = f64
        lib.orc_decode_bf16.argtypes = [ctypes.c_uint16]; lib.orc_decode_bf16.restype = f64
        lib.orc_decode_e4m3.argtypes = [ctypes.c_uint8]; lib.orc_decode_e4m3.restype = f64
        lib.orc_encode_e4m3_rne_satfinite.argtypes = [f32]
        lib.orc_encode_e4m3_rne_satfinite.restype = ctypes.c_uint8
        lib.orc_encode_f16.argtypes = [f64]; lib.orc_encode_f16.restype = ctypes.c_uint16
        lib.orc_encode_bf16.argtypes = [f64]; lib.orc_encode_bf16.restype = ctypes.c_uint16
        lib.orc_div_f32.argtypes = [f32, f32]; lib.orc_div_f32.restype = f32
        lib.orc_slot_mapping.argtypes = [P, i32, i32, P, P, i32, i32, P]
        lib.orc_slot_mapping.restype = ctypes.c_int
        lib.orc_reshape_and_cache.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i64,
                                              ctypes.c_int, ctypes.c_int, P, P]
        lib.orc_reshape_and_cache.restype = ctypes.c_int
        lib.orc_decode.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, f32,
                                   ctypes.c_int, ctypes.c_int, P, P, i32]
        lib.orc_decode.restype = ctypes.c_int
        lib.orc_chunked_prefill.argtypes = [P, P, P, i32, P, P, P, i32, P, i32, i32, i32, i32,
                                            i32, i64, f32, ctypes.c_int, ctypes.c_int, P, P]
        lib.orc_chunked_prefill.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _raw(a, dt):
    """Raw element codes of a numpy array: uint16 for 16-bit types, uint8 for E4M3."""
    want = np.uint8 if dt == "e4m3" else np.uint16
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16 and dt == "f16":
        a = a.view(np.uint16)
    if a.dtype != want:
        raise TypeError(f"expected raw {want.__name__} codes for {dt}, got {a.dtype}")
    return a


# ------------------------------------------------------------------ formats

def decode_f16(code: int) -> float:
    return _load().orc_decode_f16(int(code))


def decode_bf16(code: int) -> float:
    return _load().orc_decode_bf16(int(code))


def decode_e4m3(code: int) -> float:
    return _load().orc_decode_e4m3(int(code))


def encode_e4m3(x: float) -> int:
    return int(_load().orc_encode_e4m3_rne_satfinite(float(x)))


def encode_f16(x: float) -> int:
    return int(_load().orc_encode_f16(float(x)))


def encode_bf16(x: float) -> int:
    return int(_load().orc_encode_bf16(float(x)))


def div_f32(a: float, b: float) -> float:
    return float(_load().orc_div_f32(float(a), float(b)))


def decode_array(codes: np.ndarray, dt: str) -> np.ndarray:
    """Element-wise fp64 value of raw codes (a loop over the C decoder)."""
    lib = _load()
    fn = {"f16": lib.orc_decode_f16, "bf16": lib.orc_decode_bf16, "e4m3": lib.orc_decode_e4m3}[dt]
    flat = _raw(codes, dt).reshape(-1)
    return np.array([fn(int(c)) for c in flat], dtype=np.float64).reshape(codes.shape)


# --------------------------------------------------------------- addressing

def slot_mapping(block_tables: np.ndarray, positions: np.ndarray, block_size: int,
                 seq_ids: np.ndarray | None = None) -> np.ndarray:
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    sid = None if seq_ids is None else np.ascontiguousarray(seq_ids, dtype=np.int32)
    out = np.empty(pos.shape[0], dtype=np.int32)
    rc = _load().orc_slot_mapping(_ptr(bt), bt.shape[0], bt.shape[1], _ptr(sid), _ptr(pos),
                                  pos.shape[0], block_size, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle slot_mapping: bad table or position (rc={rc})")
    return out


# -------------------------------------------------------- reshape_and_cache

def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping_, *, block_size: int,
                      kv_dtype: str, cache_dtype: str, k_scale=None, v_scale=None) -> None:
    """In place on the numpy caches (raw codes). key/value: [T, Hkv, D]."""
    key = _raw(key, kv_dtype)
    value = _raw(value, kv_dtype)
    if not (key_cache.flags.c_contiguous and value_cache.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous")
    kc = _raw(key_cache, cache_dtype)
    vc = _raw(value_cache, cache_dtype)
    slots = np.ascontiguousarray(slot_mapping_, dtype=np.int32)
    T, Hkv, D = key.shape
    nb = kc.shape[0]
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    rc = _load().orc_reshape_and_cache(_ptr(key), _ptr(value), _ptr(kc), _ptr(vc), _ptr(slots),
                                       T, Hkv, D, block_size, nb, DTYPE_CODES[kv_dtype],
                                       DTYPE_CODES[cache_dtype], _ptr(ks), _ptr(vs))
    if rc != 0:
        raise ValueError(f"oracle reshape_and_cache failed (rc={rc})")


# ------------------------------------------------------------------- decode

def decode(query, key_cache, value_cache, block_tables, context_lens, *, scale: float,
           q_dtype: str, cache_dtype: str, k_scale=None, v_scale=None,
           partition_tokens: int = 0) -> np.ndarray:
    """fp64 output [S, H, D]. query: raw codes [S, H, D]; caches: raw codes
    [NB, BS, Hkv, D]; block_tables int32 [S, max_blocks]; context_lens int32 [S]."""
    q = _raw(query, q_dtype)
    kc = _raw(key_cache, cache_dtype)
    vc = _raw(value_cache, cache_dtype)
    if not (kc.flags.c_contiguous and vc.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous")
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, H, D = q.shape
    NB, BS, Hkv, D2 = kc.shape
    assert D2 == D and bt.shape[0] == S and cl.shape[0] == S
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    out = np.zeros((S, H, D), dtype=np.float64)
    rc = _load().orc_decode(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), bt.shape[1],
                            _ptr(cl), S, H, Hkv, D, BS, NB, float(scale),
                            DTYPE_CODES[q_dtype], DTYPE_CODES[cache_dtype], _ptr(ks), _ptr(vs),
                            int(partition_tokens))
    if rc != 0:
        raise ValueError(f"oracle decode failed (rc={rc})")
    return out


def chunked_prefill(query, key_cache, value_cache, block_tables, context_lens, cu_query_lens, *,
                    scale: float, q_dtype: str, cache_dtype: str, k_scale=None,
                    v_scale=None) -> np.ndarray:
    """fp64 output [T, H, D] of a multi-token query: rows cu_query_lens[s] ..
    cu_query_lens[s+1]-1 of query (raw codes [T, H, D]) are the last positions
    of sequence s and attend causally to its cached tokens (orc_chunked_prefill)."""
    q = _raw(query, q_dtype)
    kc = _raw(key_cache, cache_dtype)
    vc = _raw(value_cache, cache_dtype)
    if not (kc.flags.c_contiguous and vc.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous")
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    cu = np.ascontiguousarray(cu_query_lens, dtype=np.int32)
    T, H, D = q.shape
    NB, BS, Hkv, D2 = kc.shape
    S = cl.shape[0]
    assert D2 == D and bt.shape[0] == S and cu.shape[0] == S + 1
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    out = np.zeros((T, H, D), dtype=np.float64)
    rc = _load().orc_chunked_prefill(_ptr(out), _ptr(q), _ptr(cu), T, _ptr(kc), _ptr(vc),
                                     _ptr(bt), bt.shape[1], _ptr(cl), S, H, Hkv, D, BS, NB,
                                     float(scale), DTYPE_CODES[q_dtype], DTYPE_CODES[cache_dtype],
                                     _ptr(ks), _ptr(vs))
    if rc != 0:
        raise ValueError(f"oracle chunked_prefill failed (rc={rc})")
    return out


def round_to(values: np.ndarray, dt: str) -> np.ndarray:
    """Round fp64 values to f16/bf16 codes, nearest even (uint16)."""
    lib = _load()
    fn = {"f16": lib.orc_encode_f16, "bf16": lib.orc_encode_bf16}[dt]
    flat = np.asarray(values, dtype=np.float64).reshape(-1)
    return np.array([fn(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(values))


def copy_blocks(src_cache: np.ndarray, dst_cache: np.ndarray, pairs) -> None:
    """Copy whole blocks: ``dst_cache[d] = src_cache[s]`` for every (s, d) in
    ``pairs`` (block index along axis 0; the bytes are copied unchanged).

    The destinations must be distinct, and when both caches are the same array
    no destination may also be a source (each pair then reads a block no pair
    writes, so the order of the copies does not matter). Modifies ``dst_cache``.
    """
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    dsts = pairs[:, 1].tolist()
    assert len(set(dsts)) == len(dsts), "duplicate destination block"
    if src_cache is dst_cache:
        assert not set(dsts) & set(pairs[:, 0].tolist()), "a destination is also a source"
    for s, d in pairs.tolist():
        assert 0 <= s < src_cache.shape[0] and 0 <= d < dst_cache.shape[0], "block id out of range"
        dst_cache[d] = src_cache[s].copy()

