"""GPU parity: libpaged's CUDA path against the CPU oracle on the same seeded
inputs (run with -m gpu on a B200).

* reshape_and_cache: bit-exact over the whole cache (written slots and the
  untouched sentinel bytes), 16-bit copy and FP8 quantisation;
* decode: element-wise within the stated tolerance, single-pass and
  partitioned paths, all five workload shapes (reduced sizes), an edge-case
  sweep over context lengths / head_dim / block_size / query group / dtype,
  and the full-size workloads in the launch configuration the benchmark
  times, compared on sampled sequences;
* invariants on the GPU: block permutation and shared-prefix sharing give
  bit-identical outputs, repeated runs are bit-identical;
* table errors are reported through the workspace error word, never by a fault.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_448_b200 as pk
from paged_kv_cache_448_b200 import workloads as wl
from gpu_helpers import GpuStep, assert_close, dev, host_codes, i32, f32, oracle_step

pytestmark = pytest.mark.gpu


def small(cfg):
    sp = wl.spec(cfg, small=cfg != 1)
    st = wl.structure(sp)
    return sp, st, wl.host_data(sp, st)


# ------------------------------------------------------- reshape_and_cache

@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_reshape_and_cache_bit_exact(cfg):
    sp, st, hd = small(cfg)
    g = GpuStep(sp, st, hd)
    g.reshape()
    torch.cuda.synchronize()
    kc, vc, _ = oracle_step(sp, st, hd, seqs=[0])
    assert np.array_equal(host_codes(g.kc), kc)
    assert np.array_equal(host_codes(g.vc), vc)


def test_reshape_and_cache_skips_negative_slots_and_keeps_sentinel():
    rng = np.random.default_rng(3)
    T, Hkv, D, bs, NB = 50, 3, 128, 32, 9
    key = rng.integers(0, 1 << 16, (T, Hkv, D)).astype(np.uint16) & 0x7BFF  # finite f16
    val = rng.integers(0, 1 << 16, (T, Hkv, D)).astype(np.uint16) & 0x7BFF
    slots = rng.permutation(NB * bs)[:T].astype(np.int32)
    slots[::5] = -1
    kc = np.full((NB, bs, Hkv, D), 0xA5A5, np.uint16)
    vc = np.full((NB, bs, Hkv, D), 0x5A5A, np.uint16)
    gk, gv = dev(kc, "f16"), dev(vc, "f16")
    pk.reshape_and_cache(dev(key, "f16"), dev(val, "f16"), gk, gv, i32(slots))
    oracle.reshape_and_cache(key, val, kc, vc, slots, block_size=bs, kv_dtype="f16",
                             cache_dtype="f16")
    assert np.array_equal(host_codes(gk), kc) and np.array_equal(host_codes(gv), vc)


@pytest.mark.parametrize("kdt", ["f16", "bf16"])
def test_reshape_and_cache_fp8_saturates_like_the_oracle(kdt):
    rng = np.random.default_rng(4)
    T, Hkv, D, bs, NB = 33, 4, 64, 16, 5
    x = (rng.standard_normal((2, T, Hkv, D)) * 4).astype(np.float32)
    x[0, 3, 1, :5] = [1e4, -1e4, 0.0, -0.0, 3e-3]
    codes = x.astype(np.float16).view(np.uint16) if kdt == "f16" else \
        torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ks = np.array([0.004, 0.02, 0.03, 0.5], np.float32)     # some values saturate
    vs = np.array([0.01, 0.01, 0.02, 0.003], np.float32)
    slots = rng.permutation(NB * bs)[:T].astype(np.int32)
    kc = np.full((NB, bs, Hkv, D), 0x33, np.uint8)
    vc = np.full((NB, bs, Hkv, D), 0x44, np.uint8)
    gk, gv = dev(kc, "e4m3"), dev(vc, "e4m3")
    pk.reshape_and_cache(dev(codes[0], kdt), dev(codes[1], kdt), gk, gv, i32(slots),
                         k_scale=f32(ks), v_scale=f32(vs))
    oracle.reshape_and_cache(codes[0], codes[1], kc, vc, slots, block_size=bs, kv_dtype=kdt,
                             cache_dtype="e4m3", k_scale=ks, v_scale=vs)
    assert np.array_equal(host_codes(gk), kc) and np.array_equal(host_codes(gv), vc)


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("path", ["auto", "single", "split"])
def test_decode_step_matches_oracle(cfg, path):
    sp, st, hd = small(cfg)
    g = GpuStep(sp, st, hd)
    g.reshape()
    part = {"auto": None, "single": 1 << 20, "split": 4 * sp.block_size}[path]
    g.decode(partition_tokens=part)
    torch.cuda.synchronize()
    _, _, ref = oracle_step(sp, st, hd)
    assert_close(g.out_f64(), ref, sp.cache_dtype, f"cfg{cfg}/{path}")


def custom(ctxs, H, Hkv, D, bs, qdt, cdt, seed=0, spare=3):
    sp = wl.Spec("custom", len(ctxs), H, Hkv, D, bs, qdt, cdt, 1.0 / math.sqrt(D),
                 np.array(ctxs, np.int32), spare_blocks=spare, seed=seed)
    st = wl.structure(sp)
    return sp, st, wl.host_data(sp, st)


EDGE_CTX = [0, 1, 15, 16, 17, 31, 32, 33, 64, 511, 512, 513]


@pytest.mark.parametrize("qdt,cdt", [("f16", "f16"), ("bf16", "bf16"), ("bf16", "e4m3"),
                                     ("f16", "e4m3")])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
def test_decode_edge_sweep(qdt, cdt, G, D, bs):
    Hkv = 2
    sp, st, hd = custom(EDGE_CTX, Hkv * G, Hkv, D, bs, qdt, cdt, seed=G * 1000 + D + bs)
    _, _, ref = oracle_step(sp, st, hd)
    g = GpuStep(sp, st, hd)
    g.reshape()
    for part in (0, 1 << 20, 2 * bs, 5 * bs):
        g.out.fill_(float("nan"))
        g.decode(partition_tokens=part)
        torch.cuda.synchronize()
        assert_close(g.out_f64(), ref, cdt, f"{qdt}/{cdt} G{G} D{D} bs{bs} part{part}")
    assert np.all(g.out_f64()[0] == 0.0)          # context 0 -> zeros


@pytest.mark.parametrize("qdt,cdt", [("f16", "f16"), ("bf16", "bf16"), ("bf16", "e4m3")])
@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("bs", [16, 32])
def test_decode_long_partitions(qdt, cdt, G, bs):
    """Partitions longer than 512 tokens (the 4-warp CTA) with ragged tails,
    and more partitions per sequence than the short-partition sweep reaches."""
    Hkv = 2
    sp, st, hd = custom([0, 1, 600, 1100, 2049, 1056], Hkv * G, Hkv, 128, bs, qdt, cdt,
                        seed=77 + G + bs)
    _, _, ref = oracle_step(sp, st, hd)
    g = GpuStep(sp, st, hd)
    g.reshape()
    for part in (33 * bs, 48 * bs, 3 * bs):
        g.out.fill_(float("nan"))
        g.decode(partition_tokens=part)
        torch.cuda.synchronize()
        assert_close(g.out_f64(), ref, cdt, f"{qdt}/{cdt} G{G} bs{bs} part{part}")


def test_workspace_reused_across_shapes_with_garbage_partials():
    """One workspace, initialised once, then used by two partitioned launches
    of different sizes; everything past the header is garbage beforehand."""
    shapes = [custom([900, 33, 1500], 16, 2, 128, 16, "bf16", "bf16", seed=31),
              custom([700, 2000, 5, 64, 1200], 8, 8, 128, 32, "f16", "f16", seed=32)]
    ws = max((pk.decode_workspace(sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                                  sp.block_size, int(sp.context_lens.max()), 128)
              for sp, _, _ in shapes), key=lambda t: t.numel())
    ws[256:].fill_(0xFF)
    for sp, st, hd in shapes:
        _, _, ref = oracle_step(sp, st, hd)
        g = GpuStep(sp, st, hd)
        g.reshape()
        g.decode(partition_tokens=128, workspace=ws)
        torch.cuda.synchronize()
        assert_close(g.out_f64(), ref, sp.cache_dtype, f"reuse {sp.num_seqs} seqs")


def test_decode_graph_replay_is_bit_identical():
    """A captured partitioned decode (decode kernel + combine kernel, chained by
    programmatic dependent launch) replays with the same bits as the eager call."""
    sp, st, hd = small(4)
    g = GpuStep(sp, st, hd)
    g.reshape()
    ws = pk.decode_workspace(sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                             sp.block_size, g.max_ctx, 2 * sp.block_size)
    g.decode(partition_tokens=2 * sp.block_size, workspace=ws)
    torch.cuda.synchronize()
    eager = host_codes(g.out).copy()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        pk.decode(g.out, g.q, g.kc, g.vc, g.bt, g.cl, g.max_ctx, sp.scale, k_scale=g.ks,
                  v_scale=g.vs, partition_tokens=2 * sp.block_size, workspace=ws)
    for _ in range(3):
        g.out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert np.array_equal(host_codes(g.out), eager)
    pk.decode_check(ws)
    del graph


def test_decode_ignores_poisoned_slots_past_context():
    sp, st, hd = custom([5, 17, 40, 100], 8, 2, 128, 16, "bf16", "bf16", seed=9)
    for s, n in enumerate(sp.context_lens):
        if n % sp.block_size:
            b = st.block_tables[s, n // sp.block_size]
            hd.key_cache[b, n % sp.block_size:] = 0x7FC0     # NaN
            hd.value_cache[b, n % sp.block_size:] = 0xFF80   # -inf
    _, _, ref = oracle_step(sp, st, hd)
    g = GpuStep(sp, st, hd)
    g.reshape()
    g.decode()
    torch.cuda.synchronize()
    assert_close(g.out_f64(), ref, "bf16", "poisoned tail")


def test_decode_single_token_is_exactly_v0():
    sp, st, hd = custom([1, 1, 1], 4, 4, 128, 16, "f16", "f16", seed=2)
    g = GpuStep(sp, st, hd)
    g.decode()                    # no reshape: v0 is the cached row
    torch.cuda.synchronize()
    out = host_codes(g.out)
    for s in range(3):
        b = st.block_tables[s, 0]
        assert np.array_equal(out[s], hd.value_cache[b, 0])


def test_decode_invariances_on_gpu():
    sp, st, hd = small(5)
    g = GpuStep(sp, st, hd)
    g.decode()
    base = host_codes(g.out).copy()
    g.decode()
    assert np.array_equal(host_codes(g.out), base), "not deterministic"
    # permuted pool, same logical content
    pi = np.random.default_rng(1).permutation(st.num_blocks)
    kc = np.empty_like(hd.key_cache); vc = np.empty_like(hd.value_cache)
    kc[pi] = hd.key_cache; vc[pi] = hd.value_cache
    table = np.where(st.block_tables >= 0, pi[np.maximum(st.block_tables, 0)], -1)
    out = torch.empty_like(g.q)
    pk.decode(out, g.q, dev(kc, "e4m3"), dev(vc, "e4m3"), i32(table), g.cl, g.max_ctx, sp.scale,
              k_scale=g.ks, v_scale=g.vs)
    assert np.array_equal(host_codes(out), base), "block permutation changed the output"
    # private copies of the shared prefix blocks
    shared = set(np.nonzero(st.refcounts > 1)[0].tolist())
    table2, extra = st.block_tables.copy(), []
    for s in range(sp.num_seqs):
        for j in range(table2.shape[1]):
            if table2[s, j] in shared:
                extra.append(table2[s, j])
                table2[s, j] = st.num_blocks + len(extra) - 1
    kc2 = np.concatenate([hd.key_cache, hd.key_cache[extra]])
    vc2 = np.concatenate([hd.value_cache, hd.value_cache[extra]])
    pk.decode(out, g.q, dev(kc2, "e4m3"), dev(vc2, "e4m3"), i32(table2), g.cl, g.max_ctx,
              sp.scale, k_scale=g.ks, v_scale=g.vs)
    assert np.array_equal(host_codes(out), base), "private copies changed the output"


def test_bad_table_entries_are_reported_not_faulted():
    sp, st, hd = custom([40, 70], 4, 4, 128, 16, "f16", "f16", seed=5)
    g = GpuStep(sp, st, hd)
    ws = pk.decode_workspace(2, 4, 4, 128, 16, g.max_ctx)
    pk.decode_check(ws)                                  # clean
    bad = st.block_tables.copy()
    bad[1, 2] = st.num_blocks + 5                        # outside the pool
    bad[0, 0] = -4
    out = torch.empty_like(g.q)
    pk.decode(out, g.q, g.kc, g.vc, i32(bad), g.cl, g.max_ctx, sp.scale, workspace=ws)
    with pytest.raises(pk.PagedError) as e:
        pk.decode_check(ws)
    assert e.value.status == 5
    assert torch.isfinite(out.float()).all()
    pk.decode_check(ws)                                  # the word was cleared
    # a context longer than max_context_len is clipped and reported
    pk.decode(out, g.q, g.kc, g.vc, g.bt, i32([40, 300]), 70, sp.scale, workspace=ws)
    with pytest.raises(pk.PagedError):
        pk.decode_check(ws)


# ----------------------------------------------- full-size, sampled outputs

def _compact(st, seqs):
    """Blocks the sampled sequences use, renumbered densely."""
    ids = sorted({b for s in seqs for b in st.seq_block_ids[s]})
    remap = {b: i for i, b in enumerate(ids)}
    rows = [[remap[b] for b in st.seq_block_ids[s]] for s in seqs]
    mb = max(len(r) for r in rows)
    table = np.full((len(seqs), mb), -1, np.int32)
    for i, r in enumerate(rows):
        table[i, :len(r)] = r
    return np.array(ids, np.int64), table


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_size_workload_sampled(cfg):
    sp = wl.spec(cfg)
    st = wl.structure(sp)
    d = wl.device_data(sp, st)
    lens = sp.context_lens
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), sp.num_seqs // 2})
    ids, ctable = _compact(st, seqs)
    sel = torch.from_numpy(ids).cuda()
    # oracle inputs: copied before any library kernel runs
    kc_h = host_codes(d["key_cache"].index_select(0, sel))
    vc_h = host_codes(d["value_cache"].index_select(0, sel))
    q_h, nk_h, nv_h = (host_codes(d[k][seqs]) for k in ("query", "new_key", "new_value"))
    ks = None if d["k_scale"] is None else d["k_scale"].cpu().numpy()
    vs = None if d["v_scale"] is None else d["v_scale"].cpu().numpy()

    slots = pk.build_slot_mapping(st.block_tables, st.positions, sp.block_size)
    out = torch.empty_like(d["query"])
    pk.reshape_and_cache(d["new_key"], d["new_value"], d["key_cache"], d["value_cache"],
                         i32(slots), k_scale=d["k_scale"], v_scale=d["v_scale"])
    ws = pk.decode_workspace(sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                             sp.block_size, int(lens.max()), sp.partition_tokens,
                             cache_dtype=pk.dtype_code(d["key_cache"]))
    pk.decode(out, d["query"], d["key_cache"], d["value_cache"], i32(st.block_tables),
              i32(lens), int(lens.max()), sp.scale, k_scale=d["k_scale"], v_scale=d["v_scale"],
              partition_tokens=sp.partition_tokens, workspace=ws)
    pk.decode_check(ws)
    gpu = out.double().cpu().numpy()[seqs]
    assert torch.isfinite(out.float()).all()

    pos = (lens[seqs] - 1).astype(np.int32)
    oslots = oracle.slot_mapping(ctable, pos, sp.block_size)
    oracle.reshape_and_cache(nk_h, nv_h, kc_h, vc_h, oslots, block_size=sp.block_size,
                             kv_dtype=sp.q_dtype, cache_dtype=sp.cache_dtype, k_scale=ks,
                             v_scale=vs)
    # the rows the library wrote equal the oracle's, bit for bit
    assert np.array_equal(host_codes(d["key_cache"].index_select(0, sel)), kc_h)
    assert np.array_equal(host_codes(d["value_cache"].index_select(0, sel)), vc_h)
    ref = oracle.decode(q_h, kc_h, vc_h, ctable, lens[seqs], scale=np.float32(sp.scale),
                        q_dtype=sp.q_dtype, cache_dtype=sp.cache_dtype, k_scale=ks, v_scale=vs)
    assert_close(gpu, ref, sp.cache_dtype, f"full cfg{cfg} seqs {seqs}")


def _as_f32(codes: np.ndarray, dt: str) -> np.ndarray:
    if dt == "f16":
        return codes.view(np.float16).astype(np.float32)
    return (codes.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("qdt,G", [("f16", 1), ("bf16", 8)])
def test_combine_running_maximum_across_batches(qdt, G):
    """Many partitions per sequence (47 of 32 tokens), combined 16 at a time
    with a running maximum: one sequence's largest logit sits in its last
    batch of partitions (the sums so far are rescaled when it arrives), the
    other's in its first."""
    Hkv, D, bs = 2, 128, 16
    sp, st, hd = custom([1500, 1500, 700], Hkv * G, Hkv, D, bs, qdt, qdt, seed=4242 + G)
    q = _as_f32(hd.query, qdt)
    kc = hd.key_cache
    for s, t in ((0, 1490), (1, 5)):
        blk = st.block_tables[s][t // bs]
        for kvh in range(Hkv):
            # the key of token t is the group's first query head: that head's
            # logit there (about |q|^2 / sqrt(D) ~ 11) outweighs the rest by
            # ~2^16, so partitions combined before it must be rescaled
            row = q[s, kvh * G]
            kc[blk, t % bs, kvh] = wl._f32_to_codes(row.astype(np.float32), qdt)
    _, _, ref = oracle_step(sp, st, hd)
    g = GpuStep(sp, st, hd)
    g.reshape()
    g.out.fill_(float("nan"))
    g.decode(partition_tokens=2 * bs)
    torch.cuda.synchronize()
    assert_close(g.out_f64(), ref, qdt, f"{qdt} G{G} 47 partitions")
