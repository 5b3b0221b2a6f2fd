"""Seeded synthetic workloads for paged decode (inputs only).

This module generates the inputs both the CUDA path and the CPU oracle
consume: query rows, cache contents, context lengths, block tables, the new
K/V rows one decode step writes, and FP8 scales. It contains none of the
attention or indexing arithmetic: block tables are filled by handing out
physical block ids in the order of a seeded permutation of the pool, slot
mappings are NOT computed here (each side derives them itself).

Shapes follow the workloads the pages discuss:

* ``tiny``      4 sequences, contexts {1, 17, 33, 100}, 4 heads, head_dim 64,
                block_size 16, 64-block pool, fp16, scale 1/8.
* ``llama7b``   LLaMA-7B decode layer ([P4] "大模型推理KV Cache内存管理与
                PagedAttention分页显存实战": batch 32 x 2048): 32 sequences of 2048
                tokens, 32 heads, head_dim 128, block_size 16 ([P4]: 16 tokens
                per block), fp16, pool 32*128+256 blocks.
* ``llama13b_mix`` continuous-batching mix ([P2] "vLLM推理引擎架构" §3.1,
                max_num_seqs 256): 256 sequences, contexts uniform in
                [16, 4096], 40 heads, head_dim 128, bf16.
* ``gqa70b_long`` 64 query / 8 kv heads, head_dim 128, block_size 32 ([P4]:
                32 for 8K+ contexts), bf16; 8 sequences of 32768 tokens and 56
                log-uniform in [1024, 8192].
* ``prefix_fp8`` 32 groups of 4 sequences sharing a 1024-token prefix (same
                physical blocks, [P4] shared prefix with reference counts) plus
                unique suffixes uniform in [64, 512]; 32 q / 8 kv heads; E4M3
                cache with per-kv-head fp32 scales max|x|/448 of N(0,1) data
                ([P4] FP8 KV cache).

Random values: numpy PCG64 seeded with ``seed`` (default 1000 + config
number) for everything structural and for host-side data; large caches can
instead be filled on the GPU with a seeded ``torch.Generator`` (``device``
mode), which draws the same distribution but not the same numbers.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

CONFIG_NAMES = {1: "tiny", 2: "llama7b", 3: "llama13b_mix", 4: "gqa70b_long", 5: "prefix_fp8"}


@dataclasses.dataclass
class Spec:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    q_dtype: str            # "f16" | "bf16"
    cache_dtype: str        # "f16" | "bf16" | "e4m3"
    scale: float
    context_lens: np.ndarray        # int32 [S]
    shared_groups: int = 0          # prefix sharing: number of groups (0 = none)
    prefix_tokens: int = 0
    spare_blocks: int = 256
    partition_tokens: int = 0       # 0 = automatic
    seed: int = 0


@dataclasses.dataclass
class Structure:
    """Integer inputs: identical for host and device data modes."""
    num_blocks: int
    block_tables: np.ndarray        # int32 [S, max_blocks_per_seq], unused entries -1
    free_order: np.ndarray          # int32 [num_blocks]: seeded permutation of the pool
    seq_block_ids: list             # per sequence, its physical block ids
    refcounts: np.ndarray           # int32 [num_blocks]: tables referencing each block
    positions: np.ndarray           # int32 [S]: position of the token this step writes (ctx-1)


def _uniform_ints(rng, lo, hi, n):
    return rng.integers(lo, hi + 1, size=n).astype(np.int32)


def spec(config: int, seed: int | None = None, *, small: bool = False) -> Spec:
    """Spec of workload `config` (1..5). small=True shrinks it so the oracle
    finishes in about a second while keeping the shape features (several
    blocks and partitions per sequence, ragged tails, GQA groups, sharing)."""
    if seed is None:
        seed = 1000 + config
    rng = np.random.Generator(np.random.PCG64(seed))
    if config == 1:
        return Spec("tiny", 4, 4, 4, 64, 16, "f16", "f16", 1.0 / 8.0,
                    np.array([1, 17, 33, 100], np.int32), spare_blocks=0, seed=seed)
    if config == 2:
        S, ctx = (4, 700) if small else (32, 2048)
        return Spec("llama7b", S, 32, 32, 128, 16, "f16", "f16", 1.0 / math.sqrt(128),
                    np.full(S, ctx, np.int32), seed=seed)
    if config == 3:
        S, hi = (12, 1100) if small else (256, 4096)
        return Spec("llama13b_mix", S, 40, 40, 128, 16, "bf16", "bf16", 1.0 / math.sqrt(128),
                    _uniform_ints(rng, 16, hi, S), seed=seed)
    if config == 4:
        if small:
            n_long, long_len, n_short, lo, hi = 1, 2100, 3, 200, 900
        else:
            n_long, long_len, n_short, lo, hi = 8, 32768, 56, 1024, 8192
        short = np.exp(rng.uniform(math.log(lo), math.log(hi), size=n_short))
        ctx = np.concatenate([np.full(n_long, long_len), np.round(short)]).astype(np.int32)
        return Spec("gqa70b_long", len(ctx), 64, 8, 128, 32, "bf16", "bf16",
                    1.0 / math.sqrt(128), ctx, partition_tokens=512, seed=seed)
    if config == 5:
        groups, prefix, lo, hi = (3, 128, 20, 100) if small else (32, 1024, 64, 512)
        suffix = _uniform_ints(rng, lo, hi, groups * 4)
        return Spec("prefix_fp8", groups * 4, 32, 8, 128, 16, "bf16", "e4m3",
                    1.0 / math.sqrt(128), (prefix + suffix).astype(np.int32),
                    shared_groups=groups, prefix_tokens=prefix, seed=seed)
    raise ValueError(f"unknown config {config}")


# ---------------------------------------------------- multi-token queries

PREFILL_NAMES = ("chunk_llama7b", "chunk_gqa70b", "verify_gqa70b", "chunk_gqa70b_fp8")


def prefill_spec(name: str, seed: int | None = None, *, small: bool = False):
    """(Spec, query_lens) of a multi-token query workload. context_lens include
    the query tokens (its last positions); shapes follow the decode workloads:

    * ``chunk_llama7b``  chunked prefill on the LLaMA-7B shape: 16 sequences,
      a 512-token chunk after a prior context uniform in [0, 3584]; 32 heads,
      head_dim 128, block_size 16, fp16.
    * ``chunk_gqa70b``   chunked prefill on the 70B GQA shape: 16 sequences, a
      256-token chunk after a log-uniform prior context in [1024, 8192];
      64 query / 8 kv heads, block_size 32, bf16.
    * ``verify_gqa70b``  verification of 8 draft tokens for 64 sequences with
      prior contexts uniform in [1024, 4096]; 64 / 8 heads, block_size 16, bf16.
    * ``chunk_gqa70b_fp8``  ``chunk_gqa70b`` over an FP8 E4M3 cache with
      per-kv-head scales (bf16 queries), as in the prefix_fp8 decode workload.
    """
    if seed is None:
        seed = 2000 + PREFILL_NAMES.index(name)
    rng = np.random.Generator(np.random.PCG64(seed))
    if name == "chunk_llama7b":
        S, chunk, lo, hi, H, Hkv, bs, dt = (3, 40, 0, 100, 4, 4, 16, "f16") if small else \
            (16, 512, 0, 3584, 32, 32, 16, "f16")
        prior = _uniform_ints(rng, lo, hi, S)
    elif name in ("chunk_gqa70b", "chunk_gqa70b_fp8"):
        S, chunk, lo, hi, H, Hkv, bs, dt = (3, 33, 10, 150, 16, 2, 32, "bf16") if small else \
            (16, 256, 1024, 8192, 64, 8, 32, "bf16")
        prior = np.round(np.exp(rng.uniform(math.log(lo), math.log(hi), size=S))).astype(np.int32)
    elif name == "verify_gqa70b":
        S, chunk, lo, hi, H, Hkv, bs, dt = (5, 8, 5, 100, 16, 2, 16, "bf16") if small else \
            (64, 8, 1024, 4096, 64, 8, 16, "bf16")
        prior = _uniform_ints(rng, lo, hi, S)
    else:
        raise ValueError(f"unknown multi-token workload {name}")
    qlens = np.full(S, chunk, np.int32)
    sp = Spec(name, S, H, Hkv, 128, bs, dt, "e4m3" if name.endswith("_fp8") else dt,
              1.0 / math.sqrt(128), (prior + qlens).astype(np.int32), seed=seed)
    return sp, qlens


def prefill_queries_host(sp: Spec, qlens: np.ndarray) -> np.ndarray:
    """Raw codes [sum(qlens), H, D] of N(0,1) query rows."""
    rng = np.random.Generator(np.random.PCG64(sp.seed + 17))
    q = rng.standard_normal((int(qlens.sum()), sp.num_heads, sp.head_dim), dtype=np.float32)
    return _f32_to_codes(q, sp.q_dtype)


def prefill_queries_device(sp: Spec, qlens: np.ndarray, device="cuda"):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(sp.seed + 19)
    return torch.randn((int(qlens.sum()), sp.num_heads, sp.head_dim), generator=g, device=device,
                       dtype=torch.float32).to(torch_dtype(sp.q_dtype))


def prefill_flops(sp: Spec, qlens: np.ndarray) -> int:
    """Algorithmic FLOPs: every query row and head against each visible key,
    2 * head_dim for q.k and 2 * head_dim for p.v."""
    ctx = sp.context_lens.astype(np.int64)
    q = qlens.astype(np.int64)
    visible = (ctx * q - q * (q - 1) // 2).sum()    # sum over rows of (position + 1)
    return int(visible) * sp.num_heads * sp.head_dim * 4


def prefill_bytes(sp: Spec, qlens: np.ndarray) -> int:
    """Algorithmic bytes: K/V of every context token once per kv-head, the
    query rows and the output rows."""
    rows = int(qlens.sum()) * sp.num_heads * sp.head_dim * 2
    return kv_bytes(sp) + 2 * rows


def structure(sp: Spec) -> Structure:
    """Block tables from a seeded permutation of the pool: ids are handed out
    in permutation order, sequence by sequence (shared prefixes once per
    group); the pool is the blocks used plus `spare_blocks`."""
    rng = np.random.Generator(np.random.PCG64(sp.seed + 7))
    bs = sp.block_size
    ctx = sp.context_lens.astype(np.int64)
    nblk = [int(-(-int(c) // bs)) for c in ctx]
    if sp.shared_groups:
        assert sp.prefix_tokens % bs == 0
        pblk = sp.prefix_tokens // bs
        used = sp.shared_groups * pblk + sum(n - pblk for n in nblk)
    else:
        used = sum(nblk)
    num_blocks = max(used + sp.spare_blocks, 64 if sp.name == "tiny" else 1)
    order = rng.permutation(num_blocks).astype(np.int32)
    cursor = 0

    def take(n):
        nonlocal cursor
        ids = order[cursor:cursor + n]
        cursor += n
        return [int(i) for i in ids]

    seq_ids = []
    if sp.shared_groups:
        per = sp.num_seqs // sp.shared_groups
        for g in range(sp.shared_groups):
            prefix_ids = take(pblk)
            for j in range(per):
                s = g * per + j
                seq_ids.append(prefix_ids + take(nblk[s] - pblk))
    else:
        for s in range(sp.num_seqs):
            seq_ids.append(take(nblk[s]))
    mb = max(1, max(len(x) for x in seq_ids))
    table = np.full((sp.num_seqs, mb), -1, np.int32)
    refc = np.zeros(num_blocks, np.int32)
    for s, ids in enumerate(seq_ids):
        table[s, :len(ids)] = ids
        for b in ids:
            refc[b] += 1
    positions = (sp.context_lens - 1).astype(np.int32)
    return Structure(num_blocks, table, order, seq_ids, refc, positions)


# ------------------------------------------------------------------ values

def _f32_to_bf16_codes(x: np.ndarray) -> np.ndarray:
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _f32_to_codes(x: np.ndarray, dt: str) -> np.ndarray:
    if dt == "f16":
        return x.astype(np.float16).view(np.uint16)
    if dt == "bf16":
        return _f32_to_bf16_codes(x)
    raise ValueError(dt)


def _e4m3_codes(x: np.ndarray, scale_per_head: np.ndarray) -> np.ndarray:
    """Stored FP8 contents: (x / scale[h]) cast to E4M3 by torch (round to nearest)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    s = torch.from_numpy(scale_per_head.astype(np.float32)).view(1, 1, -1, 1)
    return (t / s).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@dataclasses.dataclass
class HostData:
    query: np.ndarray        # raw codes [S, H, D]
    key_cache: np.ndarray    # raw codes [NB, BS, Hkv, D]
    value_cache: np.ndarray
    new_key: np.ndarray      # raw codes [S, Hkv, D] in q dtype (the step's new token)
    new_value: np.ndarray
    k_scale: np.ndarray | None   # fp32 [Hkv] (FP8 only)
    v_scale: np.ndarray | None


def host_data(sp: Spec, st: Structure) -> HostData:
    """All values drawn on the host: N(0,1) fp32, then rounded to the storage
    type. Suited to sizes the CPU oracle handles."""
    rng = np.random.Generator(np.random.PCG64(sp.seed + 11))
    S, H, Hkv, D, BS = sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size
    q = rng.standard_normal((S, H, D), dtype=np.float32)
    kf = rng.standard_normal((st.num_blocks, BS, Hkv, D), dtype=np.float32)
    vf = rng.standard_normal((st.num_blocks, BS, Hkv, D), dtype=np.float32)
    nk = rng.standard_normal((S, Hkv, D), dtype=np.float32)
    nv = rng.standard_normal((S, Hkv, D), dtype=np.float32)
    ks = vs = None
    if sp.cache_dtype == "e4m3":
        ks = (np.abs(kf).max(axis=(0, 1, 3)) / np.float32(448.0)).astype(np.float32)
        vs = (np.abs(vf).max(axis=(0, 1, 3)) / np.float32(448.0)).astype(np.float32)
        kc, vc = _e4m3_codes(kf, ks), _e4m3_codes(vf, vs)
    else:
        kc, vc = _f32_to_codes(kf, sp.cache_dtype), _f32_to_codes(vf, sp.cache_dtype)
    return HostData(_f32_to_codes(q, sp.q_dtype), kc, vc, _f32_to_codes(nk, sp.q_dtype),
                    _f32_to_codes(nv, sp.q_dtype), ks, vs)


def torch_dtype(dt: str):
    import torch
    return {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.uint8}[dt]


def device_data(sp: Spec, st: Structure, device="cuda"):
    """Values drawn directly on the GPU with a seeded torch.Generator (for the
    full-size workloads, whose caches are GBs). Returns a dict of torch tensors
    with the same keys/shapes/dtypes as HostData (E4M3 caches as uint8)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(sp.seed + 13)
    S, H, Hkv, D, BS = sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size
    qd = torch_dtype(sp.q_dtype)
    out = {
        "query": torch.randn((S, H, D), generator=g, device=device, dtype=torch.float32).to(qd),
        "new_key": torch.randn((S, Hkv, D), generator=g, device=device, dtype=torch.float32).to(qd),
        "new_value": torch.randn((S, Hkv, D), generator=g, device=device,
                                 dtype=torch.float32).to(qd),
        "k_scale": None, "v_scale": None,
    }
    shape = (st.num_blocks, BS, Hkv, D)
    for name in ("key_cache", "value_cache"):
        if sp.cache_dtype == "e4m3":
            x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            sc = (x.abs().amax(dim=(0, 1, 3)) / 448.0).float()
            out[name] = (x / sc.view(1, 1, -1, 1)).to(torch.float8_e4m3fn).view(torch.uint8)
            out["k_scale" if name == "key_cache" else "v_scale"] = sc
            del x
        else:
            out[name] = torch.empty(shape, device=device, dtype=torch_dtype(sp.cache_dtype))
            # fill in slices to bound the fp32 temporary
            step = max(1, (1 << 26) // (BS * Hkv * D))
            for b0 in range(0, st.num_blocks, step):
                b1 = min(st.num_blocks, b0 + step)
                out[name][b0:b1] = torch.randn((b1 - b0, BS, Hkv, D), generator=g,
                                               device=device, dtype=torch.float32)
    return out


def kv_bytes(sp: Spec) -> int:
    """Algorithmic K+V bytes one decode reads: every context token's row of
    each kv-head, once for K and once for V."""
    elem = 1 if sp.cache_dtype == "e4m3" else 2
    return int(sp.context_lens.astype(np.int64).sum()) * sp.num_kv_heads * sp.head_dim * elem * 2


def decode_bytes(sp: Spec, st: Structure) -> int:
    """Algorithmic bytes of one decode: K/V rows + query + output + the block
    table entries used + context lengths."""
    qb = sp.num_seqs * sp.num_heads * sp.head_dim * 2
    used_entries = sum(len(x) for x in st.seq_block_ids)
    return kv_bytes(sp) + 2 * qb + 4 * used_entries + 4 * sp.num_seqs
