"""CPU tests of libpaged.so: it loads, exports every call include/paged.h
declares, the host allocator and table builders agree with the oracle model
bit for bit, and argument errors are rejected on the host before any launch."""
import ctypes
import os
import re

import hashlib

import numpy as np
import pytest

import oracle
from oracle.block_manager import BlockManager, OutOfBlocks
import paged_kv_cache_448_b200 as pk
from paged_kv_cache_448_b200 import _native
from paged_kv_cache_448_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "paged.h")).read()
    return sorted(set(re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", src)))


def test_library_exports_every_declared_call():
    lib = _native.lib()
    declared = header_functions()
    assert len(declared) >= 18
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(n for n, _, _ in _native.SIGNATURES) == declared


def test_library_is_the_in_tree_build():
    assert os.path.dirname(_native.LIB_PATH) == os.path.join(ROOT, "paged_kv_cache_448_b200")


# ------------------------------------------------------------- allocator

def test_allocator_matches_oracle_model_on_random_ops():
    rng = np.random.default_rng(21)
    for trial in range(20):
        nb = int(rng.integers(1, 200))
        order = rng.permutation(nb).astype(np.int32)
        ours = pk.BlockAllocator(nb, order)
        ref = BlockManager(nb, order)
        live = []                      # references held (block ids, with repeats)
        for _ in range(300):
            op = rng.integers(0, 5)
            if op == 0:
                n = int(rng.integers(0, 12))
                try:
                    expect = ref.allocate(n)
                except OutOfBlocks:
                    with pytest.raises(pk.PagedError) as ei:
                        ours.allocate(n)
                    assert ei.value.status == _native.PA_ERR_OOM
                    continue
                assert ours.allocate(n) == expect
                live.extend(expect)
            elif op == 1 and live:
                b = int(rng.choice(live))
                ref.share(b); ours.share(b)
                live.append(b)
            elif op == 2 and live:
                k = int(rng.integers(1, min(6, len(live)) + 1))
                idx = rng.choice(len(live), size=k, replace=False)
                ids = [live[i] for i in idx]
                ref.free(ids); ours.free(ids)
                for i in sorted(idx, reverse=True):
                    live.pop(i)
            elif op == 3:
                # an invalid free (a block with no references left) changes nothing
                free_ids = ref.free_blocks[:1]
                if free_ids:
                    with pytest.raises(pk.PagedError):
                        ours.free(free_ids)
            elif op == 4 and live:
                # copy-on-write of a held reference
                i = int(rng.integers(0, len(live)))
                try:
                    expect = ref.copy_on_write(live[i])
                except OutOfBlocks:
                    with pytest.raises(pk.PagedError) as ei:
                        ours.copy_on_write(live[i])
                    assert ei.value.status == _native.PA_ERR_OOM
                    continue
                assert ours.copy_on_write(live[i]) == expect
                live[i] = expect[0]
            assert ours.free_list() == ref.free_blocks
            assert ours.num_free == ref.num_free()
        for b in range(nb):
            assert ours.refcount(b) == ref.refcount[b]
        ours.close()


def test_allocator_rejects_non_permutation_and_bad_ids():
    with pytest.raises(pk.PagedError):
        pk.BlockAllocator(3, [0, 0, 1])
    a = pk.BlockAllocator(4)
    with pytest.raises(pk.PagedError):
        a.share(2)                      # free block
    ids = a.allocate(2)
    with pytest.raises(pk.PagedError):
        a.free([ids[0], ids[0]])        # more drops than references: nothing changes
    assert a.refcount(ids[0]) == 1 and a.num_free == 2
    assert a.refcount(99) == -1


def test_block_table_builder():
    t = pk.build_block_table([[5, 1], [], [3, 2, 0]], 4)
    assert t.tolist() == [[5, 1, -1, -1], [-1, -1, -1, -1], [3, 2, 0, -1]]
    with pytest.raises(pk.PagedError):
        pk.build_block_table([[1, 2, 3]], 2)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_slot_mapping_matches_oracle(cfg):
    sp = wl.spec(cfg, small=cfg != 1)
    st = wl.structure(sp)
    ours = pk.build_slot_mapping(st.block_tables, st.positions, sp.block_size)
    ref = oracle.slot_mapping(st.block_tables, st.positions, sp.block_size)
    assert np.array_equal(ours, ref)
    # every position of every sequence, with explicit sequence ids
    seq = np.concatenate([np.full(n, s, np.int32) for s, n in enumerate(sp.context_lens)])
    pos = np.concatenate([np.arange(n, dtype=np.int32) for n in sp.context_lens])
    pos[::7] = -1
    assert np.array_equal(pk.build_slot_mapping(st.block_tables, pos, sp.block_size, seq),
                          oracle.slot_mapping(st.block_tables, pos, sp.block_size, seq))


def test_slot_mapping_errors():
    t = np.array([[4, -1]], np.int32)
    with pytest.raises(pk.PagedError) as e:
        pk.build_slot_mapping(t, [20], 16)
    assert e.value.status == _native.PA_ERR_BAD_TABLE
    with pytest.raises(pk.PagedError):
        pk.build_slot_mapping(t, [40], 16)
    assert pk.build_slot_mapping(t, [-3, 3], 16, seq_ids=[0, 0]).tolist() == [-1, 67]


# --------------------------------------------------- host-side validation

def _decode_raw(**over):
    args = dict(out=16, query=16, kc=16, vc=16, bt=16, mbps=4, cl=16, max_ctx=64, S=2, H=8,
                Hkv=2, D=128, BS=16, NB=10, scale=0.1, qdt=_native.PA_F16, cdt=_native.PA_F16,
                ks=None, vs=None, part=0, ws=256, wsb=1 << 20)
    args.update(over)
    a = args
    return _native.lib().pa_decode(a["out"], a["query"], a["kc"], a["vc"], a["bt"], a["mbps"],
                                   a["cl"], a["max_ctx"], a["S"], a["H"], a["Hkv"], a["D"],
                                   a["BS"], a["NB"], a["scale"], a["qdt"], a["cdt"], a["ks"],
                                   a["vs"], a["part"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("over,status", [
    (dict(H=6, Hkv=4), _native.PA_ERR_INVALID_ARG),
    (dict(H=32, Hkv=2), _native.PA_ERR_UNSUPPORTED),        # group 16
    (dict(D=96), _native.PA_ERR_UNSUPPORTED),
    (dict(BS=8), _native.PA_ERR_UNSUPPORTED),
    (dict(qdt=_native.PA_FP8_E4M3), _native.PA_ERR_UNSUPPORTED),
    (dict(cdt=_native.PA_BF16), _native.PA_ERR_UNSUPPORTED),
    (dict(cdt=_native.PA_FP8_E4M3), _native.PA_ERR_INVALID_ARG),  # scales missing
    (dict(out=8), _native.PA_ERR_INVALID_ARG),                      # misaligned
    (dict(ws=128), _native.PA_ERR_INVALID_ARG),                     # workspace alignment
    (dict(ws=None), _native.PA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _native.PA_ERR_INVALID_ARG),
    (dict(S=-1), _native.PA_ERR_INVALID_ARG),
    (dict(NB=1 << 28), _native.PA_ERR_UNSUPPORTED),                 # pool rows > 2^31
])
def test_decode_rejects_bad_arguments_before_launch(over, status):
    assert _decode_raw(**over) == status
    assert _native.lib().pa_last_error()


def test_decode_with_no_sequences_is_a_no_op():
    assert _decode_raw(S=0, out=None, query=None) == _native.PA_OK


def test_reshape_rejects_bad_arguments():
    lib = _native.lib()
    f = lib.pa_reshape_and_cache
    ok = dict(k=16, v=16, kc=16, vc=16, sm=16, T=4, Hkv=2, D=128, BS=16, NB=4,
              kdt=_native.PA_F16, cdt=_native.PA_F16, ks=None, vs=None)

    def call(**o):
        a = dict(ok); a.update(o)
        return f(a["k"], a["v"], a["kc"], a["vc"], a["sm"], a["T"], a["Hkv"], a["D"], a["BS"],
                 a["NB"], a["kdt"], a["cdt"], a["ks"], a["vs"], None)
    assert call(D=80) == _native.PA_ERR_UNSUPPORTED
    assert call(kdt=_native.PA_FP8_E4M3) == _native.PA_ERR_UNSUPPORTED
    assert call(cdt=_native.PA_FP8_E4M3) == _native.PA_ERR_INVALID_ARG
    assert call(k=24) == _native.PA_ERR_INVALID_ARG
    assert call(T=0, k=None) == _native.PA_OK


def test_sha256_matches_fips_examples():
    import json, os
    with open(os.path.join(os.path.dirname(__file__), "golden", "sha256_fips180.json")) as f:
        vecs = json.load(f)["vectors"]
    for v in vecs:
        m = b"a" * 1000000 if v["message"] == "a*1000000" else v["message"].encode()
        assert pk.sha256(m).hex() == v["sha256"], v["cite"]
    assert pk.sha256(b"").hex() == hashlib.sha256(b"").hexdigest()
    rng = np.random.default_rng(1)
    for n in [1, 55, 56, 63, 64, 65, 119, 120, 128, 1000]:   # padding boundaries
        m = rng.integers(0, 256, n).astype(np.uint8).tobytes()
        assert pk.sha256(m) == hashlib.sha256(m).digest(), n


def test_block_hashes_match_oracle():
    from oracle.block_manager import block_hash, prompt_block_hashes
    rng = np.random.default_rng(2)
    for trial in range(20):
        bs = int(rng.choice([16, 32]))
        toks = rng.integers(-5, 200000, int(rng.integers(0, 400))).astype(np.int32)
        ours = pk.prompt_block_hashes(toks, bs)
        ref = prompt_block_hashes(toks.tolist(), bs)
        assert [bytes(r) for r in ours] == ref
    parent = bytes(rng.integers(0, 256, 32).astype(np.uint8))
    assert pk.block_hash(parent, [3, 4, 5]) == block_hash(parent, [3, 4, 5])
    assert pk.block_hash(None, []) == block_hash(None, [])


def test_prefix_cache_matches_oracle_model_on_random_requests():
    from oracle.block_manager import prompt_block_hashes
    rng = np.random.default_rng(23)
    prefixes = [rng.integers(0, 1000, 16 * int(rng.integers(1, 5))).tolist() for _ in range(4)]
    for trial in range(10):
        nb = int(rng.integers(4, 60))
        order = rng.permutation(nb).astype(np.int32)
        ours, ref = pk.BlockAllocator(nb, order), BlockManager(nb, order)
        held = []                          # block lists of live requests
        for _ in range(200):
            op = rng.integers(0, 4)
            if op <= 1:                    # a request: shared prefix + own tokens
                toks = prefixes[int(rng.integers(0, 4))] + \
                    rng.integers(0, 3, 16 * int(rng.integers(0, 3))).tolist()
                hs = prompt_block_hashes(toks, 16)
                try:
                    expect = ref.acquire_prefix(hs)
                except OutOfBlocks:
                    with pytest.raises(pk.PagedError) as ei:
                        ours.acquire_prefix(np.frombuffer(b"".join(hs), np.uint8))
                    assert ei.value.status == _native.PA_ERR_OOM
                    continue
                got = ours.acquire_prefix(np.frombuffer(b"".join(hs), np.uint8).reshape(-1, 32))
                assert got == expect
                held.append(expect[0])
            elif op == 2 and held:         # a request ends
                ids = held.pop(int(rng.integers(0, len(held))))
                ref.free(ids); ours.free(ids)
            elif op == 3 and held:         # a decode step fills a block: register it
                ids = held[int(rng.integers(0, len(held)))]
                if ids:
                    h = bytes(rng.integers(0, 256, 32).astype(np.uint8))
                    b = ids[int(rng.integers(0, len(ids)))]
                    ref.register_hash(b, h); ours.register_hash(b, h)
            assert ours.free_list() == ref.free_blocks
            for b in range(nb):
                assert ours.refcount(b) == ref.refcount[b]
            for h, b in list(ref.by_hash.items())[:8]:
                assert ours.lookup(h) == b


def test_chunked_prefill_workspace_plan():
    # chunks that fill tensor-memory CTAs, enough of them for a wave: header only
    assert pk.chunked_prefill_workspace_size(16, 16 * 512, 32, 32, 128, 512, 4096) == 256
    # one sequence's 128-token chunk (8 x 2 tcgen05 CTAs, below half a wave
    # of 148): the key range splits, partial rows for every part; its
    # 512-token chunk (8 x 16 CTAs) does not
    n = pk.chunked_prefill_workspace_size(1, 128, 32, 8, 128, 128, 8192)
    assert n > 256 and (n - 256) % (128 * 32 * (8 + 128 * 4)) < 256
    assert pk.chunked_prefill_workspace_size(1, 512, 64, 8, 128, 512, 8192) == 256
    # short chunks of many sequences already fill the GPU: no split
    assert pk.chunked_prefill_workspace_size(4096, 4096 * 8, 64, 8, 128, 8, 4096) == 256
    # few short-chunk CTAs with long contexts: partial rows for every part
    n = pk.chunked_prefill_workspace_size(16, 16 * 8, 64, 8, 128, 8, 4096)
    rows = 16 * 8 * 64
    assert n > 256 and (n - 256) % (rows * (8 + 128 * 4)) < 256
    # short chunks whose tcgen05 CTAs fill a wave (64 x 8 >= 2 per SM) run
    # there, unsplit; with 2 rows per kv-head they stay on mma.sync, split
    assert pk.chunked_prefill_workspace_size(64, 64 * 8, 64, 8, 128, 8, 4096) == 256
    assert pk.chunked_prefill_workspace_size(16, 16 * 2, 32, 32, 128, 2, 4096) > 256
    assert pk.chunked_prefill_workspace_size(64, 64 * 8, 64, 8, 64, 8, 4096) == 256
    assert pk.chunked_prefill_workspace_size(1, 1, 3, 2, 128, 1, 10) == 0   # H % Hkv != 0
    # an E4M3 cache takes tcgen05 only with head_dim 128: 4 sequences' long
    # chunks fill a tcgen05 wave (256 CTAs), unsplit, but with head_dim 64
    # they run on the mma.sync kernel, whose 1024 CTAs are split
    fp8 = _native.PA_FP8_E4M3
    assert pk.chunked_prefill_workspace_size(4, 2048, 32, 32, 128, 512, 4096, fp8) == 256
    assert pk.chunked_prefill_workspace_size(4, 2048, 32, 32, 64, 512, 4096) == 256
    assert pk.chunked_prefill_workspace_size(4, 2048, 32, 32, 64, 512, 4096, fp8) > 256
    assert pk.chunked_prefill_workspace_size(4, 2048, 32, 32, 128, 512, 4096, 7) == 0


def test_copy_blocks_rejects_bad_arguments_before_launch():
    lib = _native.lib()
    P = 1 << 20                                 # any 16-byte aligned address; never touched
    def call(src=P, sv=None, dst=P, dv=None, pairs=P, n=1, bb=4096, ns=4, nd=4, err=None):
        return lib.pa_copy_blocks(src, sv, dst, dv, pairs, n, bb, ns, nd, err, None)
    bad = _native.PA_ERR_INVALID_ARG
    assert call(n=-1) == bad
    assert call(bb=24) == bad                   # not a multiple of 16
    assert call(bb=0) == bad
    assert call(ns=0) == bad
    assert call(src=None) == bad
    assert call(pairs=None) == bad
    assert call(sv=P) == bad                    # one value cache without the other
    assert call(dst=P + 8) == bad               # misaligned
    assert call(pairs=P + 2) == bad
    assert call(n=0) == _native.PA_OK           # nothing to do, no device call


def test_chunked_prefill_rejects_bad_arguments_before_launch():
    lib = _native.lib()
    P = 1 << 20                                 # any 256-byte aligned address; never touched
    F16, BF16, E4M3 = _native.PA_F16, _native.PA_BF16, _native.PA_FP8_E4M3
    def call(T=8, mql=8, S=1, H=8, Hkv=2, D=128, bs=16, qd=BF16, cd=BF16, ks=None, vs=None,
             ws=P, wsb=256, scale=0.088, q=P, out=P, mctx=64):
        return lib.pa_chunked_prefill(out, q, P, T, mql, P, P, P, 64, P, mctx, S, H, Hkv, D, bs,
                                      64, scale, qd, cd, ks, vs, ws, wsb, None)
    bad, unsup = _native.PA_ERR_INVALID_ARG, _native.PA_ERR_UNSUPPORTED
    assert call(cd=F16) == unsup                # 16-bit cache of another dtype than the query
    assert call(qd=E4M3, cd=E4M3, ks=P, vs=P) == unsup   # the query is f16 or bf16
    assert call(cd=E4M3) == bad                 # E4M3 without its scales
    assert call(cd=E4M3, ks=P) == bad
    assert call(ks=P, vs=P) == bad              # scales with a 16-bit cache
    assert call(cd=E4M3, ks=P + 2, vs=P) == bad  # misaligned scale
    assert call(H=12) == unsup                  # group 6
    assert call(H=7) == bad                     # H % Hkv != 0
    assert call(D=96) == unsup
    assert call(bs=8) == unsup
    assert call(scale=float("nan")) == bad
    assert call(ws=None) == bad
    assert call(ws=P + 16) == bad               # not 256-byte aligned
    assert call(wsb=128) == bad                 # smaller than the header
    assert call(q=None) == bad
    assert call(out=P + 4) == bad
    assert call(T=-1) == bad
    assert call(T=0) == _native.PA_OK           # nothing to do, no device call
    # a split launch (8 tokens of one sequence over 1024 keys) needs its
    # partial rows: a workspace one vector short is refused
    need = pk.chunked_prefill_workspace_size(1, 8, 8, 2, 128, 8, 1024, BF16)
    assert need > 256
    assert call(mctx=1024, wsb=need - 16) == bad
    assert b"workspace" in lib.pa_last_error()


def test_workspace_sizes_and_partition_plan():
    # single pass: only the 256-byte header (error word and failure record)
    assert pk.decode_workspace_size(4, 4, 4, 64, 16, 100, 0) == 256
    assert pk.decode_partition_tokens(4, 4, 4, 64, 16, 100, 0) >= 100
    # forced partitions of 512 tokens over 2048: 4 partials per (seq, head)
    n = pk.decode_workspace_size(32, 32, 32, 128, 16, 2048, 512)
    rows = 32 * 32 * 4
    assert n >= 256 + rows * 8 + rows * 128 * 4
    assert pk.decode_partition_tokens(32, 32, 32, 128, 16, 2048, 512) == 512
    # partitions are whole blocks
    assert pk.decode_partition_tokens(2, 8, 8, 128, 32, 4096, 300) == 320
    # the E4M3 tcgen05 kernel (head_dim 128) wants one wave of units (two
    # CTAs per SM): 128 sequences x 8 kv-heads of up to 1534 tokens run in one
    # pass, where the 16-bit kernels cut them into 1024-token partitions;
    # with 8 sequences both cut
    fp8 = _native.PA_FP8_E4M3
    assert pk.decode_partition_tokens(128, 32, 8, 128, 16, 1534, 0, fp8) >= 1534
    assert pk.decode_workspace_size(128, 32, 8, 128, 16, 1534, 0, fp8) == 256
    assert pk.decode_partition_tokens(128, 32, 8, 128, 16, 1534, 0) == 1024
    assert pk.decode_partition_tokens(8, 32, 8, 128, 16, 1534, 0, fp8) < 1534
    # head_dim 64 over E4M3 keeps the mma.sync kernel and its plan
    assert pk.decode_partition_tokens(128, 32, 8, 64, 16, 1534, 0, fp8) == 1024


def test_slot_mapping_agrees_with_oracle_on_random_tables():
    """Property check over random tables (including -1 padding and ids near
    the int32 slot limit), positions (padding, past the table) and sequence
    ids: the library succeeds exactly when the oracle does, with equal slots."""
    from hypothesis import given, settings, strategies as st_

    @settings(max_examples=300, deadline=None, derandomize=True)
    @given(st_.data())
    def check(data):
        S = data.draw(st_.integers(1, 6))
        MB = data.draw(st_.integers(1, 6))
        bs = data.draw(st_.sampled_from([16, 32]))
        ids = st_.one_of(st_.integers(-1, 50), st_.integers(2**31 // bs - 3, 2**31 // bs + 3))
        table = np.array(data.draw(st_.lists(ids, min_size=S * MB, max_size=S * MB)),
                         np.int32).reshape(S, MB)
        n = data.draw(st_.integers(1, 12))
        pos = np.array(data.draw(st_.lists(st_.integers(-2, MB * bs + 3), min_size=n,
                                           max_size=n)), np.int32)
        sid = np.array(data.draw(st_.lists(st_.integers(0, S - 1), min_size=n, max_size=n)),
                       np.int32)
        try:
            ref = oracle.slot_mapping(table, pos, bs, sid)
        except ValueError:
            ref = None
        if ref is None:
            with pytest.raises(pk.PagedError):
                pk.build_slot_mapping(table, pos, bs, sid)
        else:
            assert np.array_equal(pk.build_slot_mapping(table, pos, bs, sid), ref)

    check()
