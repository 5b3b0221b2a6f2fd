"""GPU parity of the multi-token query path (pa_chunked_prefill) against the
oracle: the three multi-token workloads at reduced size, an edge sweep over
chunk / context lengths, head_dim, block_size, query group and dtype, a
one-token-per-sequence case against decode, error reporting, and the
full-size workloads in the launch configuration the benchmark times,
compared on sampled sequences."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_448_b200 as pk
from paged_kv_cache_448_b200 import workloads as wl
from gpu_helpers import Guarded, assert_close, dev, f32, guarded_workspace, host_codes, i32

pytestmark = pytest.mark.gpu


def run_gpu(sp, st, hd, q, qlens, table=None, ctx=None):
    """One pa_chunked_prefill call; its output and workspace sit inside guard
    bytes that must be unchanged afterwards."""
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    ctx = sp.context_lens if ctx is None else ctx
    table = st.block_tables if table is None else table
    gq = dev(q, sp.q_dtype)
    out_g = Guarded(tuple(gq.shape), gq.dtype, fill=float("nan"))
    out = out_g.t
    kc, vc = dev(hd.key_cache, sp.cache_dtype), dev(hd.value_cache, sp.cache_dtype)
    ws_g = guarded_workspace(pk.chunked_prefill_workspace_size(
        sp.num_seqs, int(qlens.sum()), sp.num_heads, sp.num_kv_heads, sp.head_dim,
        int(qlens.max()), int(np.max(ctx)), pk.dtype_code(kc)))
    ws = ws_g.t
    pk.chunked_prefill(out, gq, i32(cu), int(qlens.max()), kc, vc, i32(table), i32(ctx),
                       int(np.max(ctx)), sp.scale, k_scale=f32(hd.k_scale),
                       v_scale=f32(hd.v_scale), workspace=ws)
    torch.cuda.synchronize()
    out_g.check("multi-token output")
    ws_g.check("multi-token workspace")
    return out, ws, cu


def run_oracle(sp, st, hd, q, cu, table=None, ctx=None):
    return oracle.chunked_prefill(q, hd.key_cache, hd.value_cache,
                                  st.block_tables if table is None else table,
                                  sp.context_lens if ctx is None else ctx, cu,
                                  scale=np.float32(sp.scale), q_dtype=sp.q_dtype,
                                  cache_dtype=sp.cache_dtype, k_scale=hd.k_scale,
                                  v_scale=hd.v_scale)


@pytest.mark.parametrize("name", wl.PREFILL_NAMES)
def test_multi_token_workloads_small(name):
    sp, qlens = wl.prefill_spec(name, small=True)
    st = wl.structure(sp)
    hd = wl.host_data(sp, st)
    q = wl.prefill_queries_host(sp, qlens)
    out, ws, cu = run_gpu(sp, st, hd, q, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, q, cu), sp.cache_dtype, name)


def custom(ctxs, qlens, H, Hkv, D, bs, dt, seed, cache_dt=None):
    sp = wl.Spec("custom", len(ctxs), H, Hkv, D, bs, dt, cache_dt or dt, 1.0 / math.sqrt(D),
                 np.array(ctxs, np.int32), spare_blocks=3, seed=seed)
    st = wl.structure(sp)
    hd = wl.host_data(sp, st)
    q = wl.prefill_queries_host(sp, np.array(qlens, np.int32))
    return sp, st, hd, q, np.array(qlens, np.int32)


# Chunk lengths that cross CTA row tiles and 16-token K tiles, with a full
# prefill (q_len == ctx), single tokens and a one-token context. The launch
# picks the kernel by max_query_len x group: >= 128 rows fill a tensor-memory
# (tcgen05) CTA, fewer run on the 64-row mma.sync kernel; each set below
# reaches one of them for every group size.
EDGE = {
    "tcgen05": ([1, 17, 40, 200, 33, 150, 130], [1, 17, 9, 150, 1, 129, 65]),
    "mma_sync": ([1, 17, 40, 100, 9], [1, 15, 9, 8, 9]),
}


@pytest.mark.parametrize("kernel", ["tcgen05", "mma_sync"])
@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
def test_multi_token_edge_sweep(kernel, dt, G, D, bs):
    ctxs, qlens = EDGE[kernel]
    assert (max(qlens) * G >= 128) == (kernel == "tcgen05")
    sp, st, hd, q, qlens = custom(ctxs, qlens, 2 * G, 2, D, bs, dt, seed=G * 100 + D + bs)
    out, ws, cu = run_gpu(sp, st, hd, q, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, q, cu), dt,
                 f"{dt} G{G} D{D} bs{bs}")


@pytest.mark.parametrize("chunks", ["tcgen05", "mma_sync"])
@pytest.mark.parametrize("qdt", ["f16", "bf16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
def test_multi_token_e4m3_cache(chunks, qdt, G, D, bs):
    """An E4M3 cache with per-kv-head scales, both chunk sets of the edge
    sweep: long chunks with head_dim 128 on tcgen05 (kind::f8f6f4), the rest
    on the mma.sync kernel."""
    ctxs, qlens = EDGE[chunks]
    sp, st, hd, q, qlens = custom(ctxs, qlens, 2 * G, 2, D, bs, qdt, seed=G * 10 + D + bs + 7,
                                  cache_dt="e4m3")
    out, ws, cu = run_gpu(sp, st, hd, q, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, q, cu), "e4m3",
                 f"e4m3 {qdt} G{G} D{D} bs{bs}")


@pytest.mark.parametrize("cache", ["bf16", "e4m3"])
@pytest.mark.parametrize("G,q", [(4, 8), (8, 1), (8, 5)])
def test_short_chunks_of_many_sequences_on_tcgen05(cache, G, q):
    """Short chunks (fewer than 128 rows per kv-head) whose tcgen05 CTAs fill
    a wave run there, unsplit: 150 sequences x 2 kv-heads, ragged chunks of at
    most q tokens, contexts long enough that the mma.sync kernel would split."""
    rng = np.random.default_rng(40 + G + q)
    n = 150
    ctxs = rng.integers(1, 700, size=n)
    ctxs[:3] = [1, 699, 520]
    qlens = np.minimum(rng.integers(1, q + 1, size=n), ctxs)
    qlens[1] = q
    sp, st, hd, qv, qlens = custom(list(ctxs), list(qlens), 2 * G, 2, 128, 16, "bf16",
                                   seed=70 + G + q, cache_dt=cache)
    code = pk._native.PA_FP8_E4M3 if cache == "e4m3" else pk._native.PA_BF16
    assert pk.chunked_prefill_workspace_size(n, int(qlens.sum()), 2 * G, 2, 128, q, 699,
                                             code) == 256
    out, ws, cu = run_gpu(sp, st, hd, qv, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, qv, cu), cache,
                 f"short chunks {cache} G{G} q{q}")


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("G", [1, 2])
@pytest.mark.parametrize("D", [64, 128])
def test_short_units_with_rows_held_twice(dt, G, D):
    """Units of at most 64 rows on tcgen05 hold each row in two lanes, which
    take the lower and the upper 32 tokens of every 64-token step and are
    merged at the end. 150 sequences x 2 kv-heads fill the kernel's wave; the
    chunks reach 64 rows per unit (64 / G tokens), and the contexts sit on
    both sides of the half-step and step boundaries (a copy that sees no
    token at all, a last step that one copy only reaches)."""
    rng = np.random.default_rng(300 + 10 * G + D)
    n = 150
    qmax = 64 // G
    ctxs = rng.integers(1, 400, size=n)
    ctxs[:10] = [1, 31, 32, 33, 63, 64, 65, 95, 96, 97]
    qlens = np.minimum(rng.integers(1, qmax + 1, size=n), ctxs)
    qlens[6] = qmax  # contexts of 65 and 97 tokens: full-length chunks
    qlens[9] = qmax
    sp, st, hd, qv, qlens = custom(list(ctxs), list(qlens), 2 * G, 2, D, 16, dt,
                                   seed=310 + 10 * G + D)
    assert int(qlens.max()) * G == 64
    out, ws, cu = run_gpu(sp, st, hd, qv, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, qv, cu), dt,
                 f"rows held twice {dt} G{G} D{D}")


@pytest.mark.parametrize("n,equal", [(256, False), (257, False), (300, True), (40, True)])
def test_units_in_launch_order_cover_every_row(n, equal):
    """The tcgen05 CTAs take their units longest context first (each CTA ranks
    the sequences by context length) up to 256 sequences, in index order above.
    Both sides of that bound, and contexts that all tie (ranks broken by
    index), must still give every row exactly once: the output starts as NaN
    and is compared whole. The 40-sequence case has 300-token chunks over two
    row groups (three query tiles per sequence, the last one first)."""
    rng = np.random.default_rng(90 + n)
    if n == 40:
        G, D = 2, 128
        ctxs = np.full(n, 400)
        qlens = rng.integers(1, 301, size=n)
        qlens[0] = 300
    else:
        G, D = 8, 64
        ctxs = np.full(n, 180) if equal else rng.integers(1, 300, size=n)
        qlens = np.minimum(rng.integers(1, 9, size=n), ctxs)
        qlens[0] = 8
    sp, st, hd, qv, qlens = custom(list(ctxs), list(qlens), 2 * G, 2, D, 16, "f16",
                                   seed=80 + n)
    out, ws, cu = run_gpu(sp, st, hd, qv, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, qv, cu), "f16",
                 f"launch order n{n} equal={equal}")


@pytest.mark.parametrize("qdt,cache,G,D,bs,qlens", [
    ("bf16", "bf16", 8, 128, 16, [150, 129, 140]),   # two row groups (>= 256 rows)
    ("f16", "f16", 2, 128, 16, [200, 150, 131]),     # two groups, f16: rows held whole
    ("bf16", "e4m3", 8, 128, 32, [100, 70, 65]),     # two groups over an E4M3 cache
    ("f16", "f16", 1, 128, 32, [200, 129, 160]),     # one row group
    ("bf16", "e4m3", 4, 128, 16, [64, 40, 33]),
    ("f16", "f16", 2, 64, 32, [100, 70, 65]),
])
def test_split_key_range_tcgen05(qdt, cache, G, D, bs, qlens):
    """Long chunks of three sequences: too few tcgen05 CTAs for a wave, so
    each key range is cut into parts merged by the combine kernel; rows
    whose causal range ends inside an earlier part, ragged last parts."""
    ctxs = [2100, 700, 3333]
    sp, st, hd, q, qlens = custom(ctxs, qlens, 2 * G, 2, D, bs, qdt, seed=990 + G + D,
                                  cache_dt=cache)
    code = {"f16": 0, "bf16": 1, "e4m3": 2}[cache]
    assert max(qlens) * G >= 128
    assert pk.chunked_prefill_workspace_size(3, int(qlens.sum()), 2 * G, 2, D, int(qlens.max()),
                                             3333, code) > 256
    out, ws, cu = run_gpu(sp, st, hd, q, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, q, cu), cache,
                 f"tcgen05 split {cache} G{G} D{D}")


@pytest.mark.parametrize("qdt,G,D,bs", [("bf16", 8, 128, 16), ("f16", 2, 64, 32)])
def test_split_key_range_e4m3(qdt, G, D, bs):
    ctxs, qlens = [2100, 700, 3333], [8, 5, 8]
    sp, st, hd, q, qlens = custom(ctxs, qlens, 2 * G, 2, D, bs, qdt, seed=950 + G,
                                  cache_dt="e4m3")
    assert pk.chunked_prefill_workspace_size(3, sum(qlens), 2 * G, 2, D, 8, 3333,
                                             pk._native.PA_FP8_E4M3) > 256
    out, ws, cu = run_gpu(sp, st, hd, q, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, q, cu), "e4m3",
                 f"split e4m3 {qdt} G{G}")


@pytest.mark.parametrize("dt,G,D,bs", [("bf16", 8, 128, 16), ("f16", 4, 64, 32),
                                       ("bf16", 2, 128, 32), ("f16", 1, 128, 16)])
def test_split_key_range_for_short_chunks(dt, G, D, bs):
    """Few CTAs (short chunks, few sequences and kv-heads) and long contexts:
    the key range is cut into parts combined by a second kernel; ragged last
    parts, rows whose causal range ends inside an earlier part."""
    ctxs, qlens = [2100, 700, 3333], [8, 5, 8]
    assert max(qlens) * G < 128
    assert pk.chunked_prefill_workspace_size(3, sum(qlens), 2 * G, 2, D, 8, 3333) > 256
    sp, st, hd, q, qlens = custom(ctxs, qlens, 2 * G, 2, D, bs, dt, seed=900 + G)
    out, ws, cu = run_gpu(sp, st, hd, q, qlens)
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), run_oracle(sp, st, hd, q, cu), dt,
                 f"split {dt} G{G} D{D} bs{bs}")


def test_one_token_per_sequence_matches_decode_and_oracle():
    sp, st, hd, q, qlens = custom([5, 64, 300, 1], [1, 1, 1, 1], 16, 2, 128, 16, "bf16", seed=5)
    out, ws, cu = run_gpu(sp, st, hd, q, qlens)
    ref = run_oracle(sp, st, hd, q, cu)
    assert_close(out.double().cpu().numpy(), ref, "bf16", "one token")
    dout = torch.empty_like(out)
    pk.decode(dout, dev(q, "bf16"), dev(hd.key_cache, "bf16"), dev(hd.value_cache, "bf16"),
              i32(st.block_tables), i32(sp.context_lens), int(sp.context_lens.max()), sp.scale)
    assert_close(dout.double().cpu().numpy(), ref, "bf16", "decode")


def test_errors_are_reported_not_faulted():
    sp, st, hd, q, qlens = custom([40, 70], [40, 10], 8, 2, 128, 16, "f16", seed=6)
    bad = st.block_tables.copy()
    bad[1, 1] = st.num_blocks + 9                 # outside the pool: read as zeros
    out, ws, cu = run_gpu(sp, st, hd, q, qlens, table=bad)
    with pytest.raises(pk.PagedError) as e:
        pk.decode_check(ws)
    assert e.value.status == 5
    assert torch.isfinite(out.float()).all()
    # a chunk longer than its context: its rows are zeros, the rest is right
    ctx = np.array([30, 70], np.int32)
    out, ws, cu = run_gpu(sp, st, hd, q, qlens, ctx=ctx)
    with pytest.raises(pk.PagedError):
        pk.decode_check(ws)
    o = out.double().cpu().numpy()
    assert np.all(o[:40] == 0.0)
    ref = oracle.chunked_prefill(q[40:], hd.key_cache, hd.value_cache, st.block_tables[1:],
                                 ctx[1:], np.array([0, 10], np.int32), scale=np.float32(sp.scale),
                                 q_dtype="f16", cache_dtype="f16")
    assert_close(o[40:], ref, "f16", "second sequence")


def test_block_permutation_keeps_the_bits():
    sp, st, hd, q, qlens = custom([90, 45], [50, 45], 8, 8, 64, 16, "bf16", seed=7)
    base, _, cu = run_gpu(sp, st, hd, q, qlens)
    pi = np.random.default_rng(1).permutation(st.num_blocks)
    kc = np.empty_like(hd.key_cache); vc = np.empty_like(hd.value_cache)
    kc[pi] = hd.key_cache; vc[pi] = hd.value_cache
    table = np.where(st.block_tables >= 0, pi[np.maximum(st.block_tables, 0)], -1)
    hd2 = wl.HostData(hd.query, kc, vc, hd.new_key, hd.new_value, None, None)
    out, _, _ = run_gpu(sp, st, hd2, q, qlens, table=table.astype(np.int32))
    assert np.array_equal(host_codes(out), host_codes(base))


@pytest.mark.parametrize("name", wl.PREFILL_NAMES)
def test_multi_token_full_size_sampled(name):
    """Full-size workload in the benchmark's launch configuration; the oracle
    checks the shortest sequence's rows (and the longest's last chunk rows
    for the verification workload, whose chunks are short)."""
    sp, qlens = wl.prefill_spec(name)
    st = wl.structure(sp)
    d = wl.device_data(sp, st)
    q = wl.prefill_queries_device(sp, qlens)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    out = torch.empty_like(q)
    ws = pk.chunked_prefill_workspace(sp.num_seqs, int(qlens.sum()), sp.num_heads,
                                      sp.num_kv_heads, sp.head_dim, int(qlens.max()),
                                      int(sp.context_lens.max()), pk.dtype_code(d["key_cache"]))
    pk.chunked_prefill(out, q, i32(cu), int(qlens.max()), d["key_cache"], d["value_cache"],
                       i32(st.block_tables), i32(sp.context_lens), int(sp.context_lens.max()),
                       sp.scale, k_scale=d["k_scale"], v_scale=d["v_scale"], workspace=ws)
    pk.decode_check(ws)
    assert torch.isfinite(out.float()).all()
    picks = [int(np.argmin(sp.context_lens))]
    if name == "verify_gqa70b":
        picks.append(int(np.argmax(sp.context_lens)))
    for s in picks:
        ids = st.seq_block_ids[s]
        sel = torch.tensor(ids, device="cuda")
        kc = host_codes(d["key_cache"].index_select(0, sel))
        vc = host_codes(d["value_cache"].index_select(0, sel))
        table = np.arange(len(ids), dtype=np.int32)[None, :]
        qs = host_codes(q[cu[s]:cu[s + 1]])
        ks, vs = (None, None) if d["k_scale"] is None else \
            (d["k_scale"].cpu().numpy(), d["v_scale"].cpu().numpy())
        ref = oracle.chunked_prefill(qs, kc, vc, table, sp.context_lens[[s]],
                                     np.array([0, qlens[s]], np.int32), scale=np.float32(sp.scale),
                                     q_dtype=sp.q_dtype, cache_dtype=sp.cache_dtype,
                                     k_scale=ks, v_scale=vs)
        assert_close(out[cu[s]:cu[s + 1]].double().cpu().numpy(), ref, sp.cache_dtype,
                     f"{name} seq {s}")
