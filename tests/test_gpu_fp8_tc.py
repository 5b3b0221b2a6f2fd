"""GPU parity of the decode over an E4M3 cache with head_dim 128, which runs
on the tcgen05 kernel with the tokens on M (128-token tiles), against the
oracle: contexts around the 128-token tile boundaries with ragged blocks,
every query group and both block sizes, single pass and partitions; a running
maximum that grows by more than the lazy margin from tile to tile (so the
output accumulator in tensor memory is rescaled); NaN codes in the cache rows
past each context (they must not reach the output); and the first tile of a
unit that is also its last."""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_448_b200 import workloads as wl
from gpu_helpers import GpuStep, assert_close, oracle_step

pytestmark = pytest.mark.gpu

TILE_CTX = [1, 127, 128, 129, 255, 256, 257, 383, 1000, 1536]


def custom(ctxs, H, Hkv, bs, qdt, seed, spare=3):
    sp = wl.Spec("fp8tc", len(ctxs), H, Hkv, 128, bs, qdt, "e4m3", 1.0 / math.sqrt(128),
                 np.array(ctxs, np.int32), spare_blocks=spare, seed=seed)
    st = wl.structure(sp)
    return sp, st, wl.host_data(sp, st)


@pytest.mark.parametrize("qdt", ["bf16", "f16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [16, 32])
def test_fp8_decode_tile_boundaries(qdt, G, bs):
    Hkv = 2
    sp, st, hd = custom(TILE_CTX, Hkv * G, Hkv, bs, qdt, seed=300 + G * 10 + bs)
    _, _, ref = oracle_step(sp, st, hd)
    g = GpuStep(sp, st, hd)
    g.reshape()
    for part in (0, 1 << 20, 8 * bs, 16 * bs, 3 * bs):
        g.out.fill_(float("nan"))
        g.decode(partition_tokens=part)
        assert_close(g.out_f64(), ref, "e4m3", f"{qdt} G{G} bs{bs} part{part}", out_dtype=qdt)


def _set_rows(cache, st, s, t0, t1, bs, code):
    for t in range(t0, t1):
        cache[st.block_tables[s, t // bs], t % bs] = code


@pytest.mark.parametrize("G", [1, 4, 8])
def test_fp8_decode_maximum_growing_across_tiles(G):
    """Keys equal to the query direction with a magnitude that doubles every
    128 tokens: each tile's logits pass the running maximum by more than the
    lazy margin (base 2), so O is rescaled after every tile, and the softmax
    ends up concentrated on the last tile."""
    Hkv, bs = 2, 16
    ctxs = [600, 130, 384]
    sp, st, hd = custom(ctxs, Hkv * G, Hkv, bs, "bf16", seed=41 + G)
    hd.k_scale[:] = 1.0
    one = np.uint16(0x3F80)                         # bf16 1.0
    hd.query[:] = one
    for s, n in enumerate(ctxs):
        for i, t0 in enumerate(range(0, n, 128)):
            code = oracle.encode_e4m3(0.25 * 2.0 ** i)
            _set_rows(hd.key_cache, st, s, t0, min(n, t0 + 128), bs, code)
    # the step's new token (written by reshape_and_cache) continues the pattern
    last = [(n - 1) // 128 for n in ctxs]
    for s in range(len(ctxs)):   # bf16 code of a power of two: the top half of its fp32 bits
        hd.new_key[s] = np.uint16(np.float32(0.25 * 2.0 ** last[s]).view(np.uint32) >> 16)
    _, _, ref = oracle_step(sp, st, hd)
    g = GpuStep(sp, st, hd)
    g.reshape()
    for part in (0, 1 << 20, 256):
        g.out.fill_(float("nan"))
        g.decode(partition_tokens=part)
        assert_close(g.out_f64(), ref, "e4m3", f"G{G} part{part}", out_dtype="bf16")


@pytest.mark.parametrize("G", [2, 8])
def test_fp8_decode_ignores_nan_codes_past_context(G):
    """Rows after each context in its last block hold E4M3 NaN codes (0x7F,
    0xFF) in K and V; blocks past the context are never read."""
    Hkv, bs = 2, 32
    ctxs = [5, 129, 300, 33, 640]
    sp, st, hd = custom(ctxs, Hkv * G, Hkv, bs, "bf16", seed=51 + G)
    for s, n in enumerate(ctxs):
        if n % bs:
            b = st.block_tables[s, n // bs]
            hd.key_cache[b, n % bs:] = 0x7F
            hd.value_cache[b, n % bs:] = 0xFF
    # positions n-1 are rewritten by the step's reshape: keep the poison after them
    _, _, ref = oracle_step(sp, st, hd)
    assert np.isfinite(ref).all()
    g = GpuStep(sp, st, hd)
    g.reshape()
    for part in (0, 1 << 20, 64):
        g.out.fill_(float("nan"))
        g.decode(partition_tokens=part)
        assert_close(g.out_f64(), ref, "e4m3", f"G{G} part{part}", out_dtype="bf16")
