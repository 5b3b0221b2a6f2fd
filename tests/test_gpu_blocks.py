"""GPU parity of whole-block copies (pa_copy_blocks) against the oracle:
copy-on-write inside a cache, copies between caches, migration to and from a
pinned host pool, and copy-on-write followed by a write and a decode step.
Every comparison is bit-exact over the whole destination cache."""
import numpy as np
import pytest
import torch

import oracle
from oracle.block_manager import BlockManager
import paged_kv_cache_448_b200 as pk
from paged_kv_cache_448_b200 import workloads as wl
from gpu_helpers import GpuStep, assert_close, dev, host_codes, i32

pytestmark = pytest.mark.gpu

# (block_size, num_kv_heads, head_dim, dtype): 2 KB (part of one 32 KB chunk),
# 32 KB (exactly one), 128 KB (four), 160 KB (five)
SHAPES = [(16, 1, 64, "f16"), (32, 8, 128, "e4m3"), (16, 32, 128, "f16"), (16, 40, 128, "bf16")]


def _codes(rng, shape, dt):
    if dt == "e4m3":
        return rng.integers(0, 256, shape).astype(np.uint8)
    return rng.integers(0, 1 << 16, shape).astype(np.uint16)


def _pairs(rng, nb, n):
    """n pairs whose destinations are distinct and never a source."""
    perm = rng.permutation(nb)
    return np.stack([perm[:n], perm[n:2 * n]], 1).astype(np.int32)


@pytest.mark.parametrize("bs,hkv,d,dt", SHAPES)
def test_copy_within_a_cache_is_bit_exact(bs, hkv, d, dt):
    rng = np.random.default_rng(bs * 1000 + hkv + d)
    nb = 37
    k = _codes(rng, (nb, bs, hkv, d), dt)
    v = _codes(rng, (nb, bs, hkv, d), dt)
    pairs = _pairs(rng, nb, 11)
    gk, gv = dev(k, dt), dev(v, dt)
    pk.copy_blocks(gk, gv, gk, gv, i32(pairs))
    oracle.copy_blocks(k, k, pairs)
    oracle.copy_blocks(v, v, pairs)
    torch.cuda.synchronize()
    assert np.array_equal(host_codes(gk), k) and np.array_equal(host_codes(gv), v)


@pytest.mark.parametrize("bs,hkv,d,dt", SHAPES)
def test_copy_between_caches_key_only(bs, hkv, d, dt):
    rng = np.random.default_rng(7 + d)
    src = _codes(rng, (20, bs, hkv, d), dt)
    dst = np.full((9, bs, hkv, d), 0x5A, src.dtype)
    pairs = np.stack([rng.permutation(20)[:9], rng.permutation(9)], 1).astype(np.int32)
    gs, gd = dev(src, dt), dev(dst, dt)
    pk.copy_blocks(gs, None, gd, None, i32(pairs))
    oracle.copy_blocks(src, dst, pairs)
    torch.cuda.synchronize()
    assert np.array_equal(host_codes(gd), dst)
    assert np.array_equal(host_codes(gs), src)


def test_out_of_range_pairs_are_skipped_and_reported():
    rng = np.random.default_rng(3)
    k = _codes(rng, (8, 16, 2, 64), "f16")
    v = _codes(rng, (8, 16, 2, 64), "f16")
    pairs = np.array([[0, 5], [9, 6], [1, -1], [2, 7]], np.int32)
    gk, gv = dev(k, "f16"), dev(v, "f16")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.copy_blocks(gk, gv, gk, gv, i32(pairs), error_word=err)
    oracle.copy_blocks(k, k, pairs[[0, 3]])
    oracle.copy_blocks(v, v, pairs[[0, 3]])
    torch.cuda.synchronize()
    assert int(err.item()) & 1
    assert np.array_equal(host_codes(gk), k) and np.array_equal(host_codes(gv), v)


def test_swap_out_to_pinned_host_and_back():
    rng = np.random.default_rng(11)
    bs, hkv, d = 16, 8, 128
    k = _codes(rng, (64, bs, hkv, d), "bf16")
    v = _codes(rng, (64, bs, hkv, d), "bf16")
    gk, gv = dev(k, "bf16"), dev(v, "bf16")
    hk = torch.zeros((24, bs, hkv, d), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    out_pairs = np.stack([rng.permutation(64)[:20], rng.permutation(24)[:20]], 1).astype(np.int32)
    pk.copy_blocks(gk, gv, hk, hv, i32(out_pairs))
    torch.cuda.synchronize()
    ek, ev = np.zeros((24, bs, hkv, d), np.uint16), np.zeros((24, bs, hkv, d), np.uint16)
    oracle.copy_blocks(k, ek, out_pairs)
    oracle.copy_blocks(v, ev, out_pairs)
    assert np.array_equal(host_codes(hk), ek) and np.array_equal(host_codes(hv), ev)
    # back into other device blocks; the pairs themselves live in pinned memory
    in_pairs = np.stack([out_pairs[:, 1], rng.permutation(64)[:20]], 1).astype(np.int32)
    pp = torch.from_numpy(in_pairs).pin_memory()
    pk.copy_blocks(hk, hv, gk, gv, pp)
    torch.cuda.synchronize()
    oracle.copy_blocks(ek, k, in_pairs)
    oracle.copy_blocks(ev, v, in_pairs)
    assert np.array_equal(host_codes(gk), k) and np.array_equal(host_codes(gv), v)
    # pageable host memory has no device address: refused before any launch
    with pytest.raises(pk.PagedError):
        pk.copy_blocks(gk, gv, torch.zeros(hk.shape, dtype=hk.dtype),
                       torch.zeros(hv.shape, dtype=hv.dtype), i32(out_pairs))


def test_copy_on_write_then_write_then_decode():
    """A shared prefix block is made private for one sequence (allocator +
    copy), a token inside it is rewritten through reshape_and_cache, and the
    decode step matches the oracle running the same three steps; the other
    sequences' outputs keep their bits."""
    sp = wl.spec(5, small=True)
    st = wl.structure(sp)
    hd = wl.host_data(sp, st)
    g = GpuStep(sp, st, hd)
    g.decode()
    before = host_codes(g.out).copy()

    alloc = pk.BlockAllocator(st.num_blocks, st.free_order)
    ref = BlockManager(st.num_blocks, st.free_order)
    pblk = sp.prefix_tokens // sp.block_size
    per = sp.num_seqs // sp.shared_groups
    for grp in range(sp.shared_groups):
        for m in (alloc, ref):
            prefix = m.allocate(pblk)
            for _ in range(per - 1):
                for b in prefix:
                    m.share(b)
            for j in range(per):
                m.allocate(len(st.seq_block_ids[grp * per + j]) - pblk)
    s0, j = per + 1, pblk - 1                   # a member of group 1, last prefix block
    old = int(st.block_tables[s0, j])
    new, must_copy = alloc.copy_on_write(old)
    assert (new, must_copy) == ref.copy_on_write(old) and must_copy
    pairs = np.array([[old, new]], np.int32)
    pk.copy_blocks(g.kc, g.vc, g.kc, g.vc, i32(pairs))
    kc, vc = hd.key_cache.copy(), hd.value_cache.copy()
    oracle.copy_blocks(kc, kc, pairs)
    oracle.copy_blocks(vc, vc, pairs)
    table = st.block_tables.copy()
    table[s0, j] = new
    g.bt = i32(table)
    # rewrite position j*bs + 5 of s0 with the step's new K/V row of s0
    pos = np.array([j * sp.block_size + 5], np.int32)
    slot = pk.build_slot_mapping(table[[s0]], pos, sp.block_size)
    assert slot[0] == new * sp.block_size + 5
    pk.reshape_and_cache(g.nk[[s0]], g.nv[[s0]], g.kc, g.vc, i32(slot), k_scale=g.ks,
                         v_scale=g.vs)
    oracle.reshape_and_cache(hd.new_key[[s0]], hd.new_value[[s0]], kc, vc, slot,
                             block_size=sp.block_size, kv_dtype=sp.q_dtype,
                             cache_dtype=sp.cache_dtype, k_scale=hd.k_scale, v_scale=hd.v_scale)
    torch.cuda.synchronize()
    assert np.array_equal(host_codes(g.kc), kc) and np.array_equal(host_codes(g.vc), vc)
    g.decode()
    torch.cuda.synchronize()
    out = host_codes(g.out)
    others = [s for s in range(sp.num_seqs) if s != s0]
    assert np.array_equal(out[others], before[others])
    refout = oracle.decode(hd.query, kc, vc, table, sp.context_lens, scale=np.float32(sp.scale),
                           q_dtype=sp.q_dtype, cache_dtype=sp.cache_dtype, k_scale=hd.k_scale,
                           v_scale=hd.v_scale)
    assert_close(g.out_f64(), refout, sp.cache_dtype, "copy-on-write step")
