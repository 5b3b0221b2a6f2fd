"""Failure detection on the GPU without a fault: every pipeline wait of the
decode and multi-token kernels is bounded by wall time. pa_inject_wait_timeout
makes the next launch leave out the loads of one tile of its first CTA and
bounds its waits by a short limit; the wait for that tile then runs out. The
kernel must record the failure (site and CTA), set the timeout bit that the
check call reports as PA_ERR_CUDA, let its loads (and, on tcgen05, its MMAs)
in flight complete before its shared and tensor memory go away, and leave
zeros (or an empty partial) for the rows it could not finish. Every other row
must still match the oracle, and a clean call right after on the same stream
must pass parity: the context stays usable.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_448_b200 as pk
from paged_kv_cache_448_b200 import _native
from paged_kv_cache_448_b200 import workloads as wl
from gpu_helpers import GpuStep, assert_close, dev, f32, i32

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000  # 20 ms: far above any real load latency, keeps the test short


def _expect_timeout(check, site):
    with pytest.raises(pk.PagedError) as e:
        check()
    msg = str(e.value)
    assert e.value.status == _native.PA_ERR_CUDA, msg
    assert "timed out" in msg and f"site {site} " in msg and "CTA (0, 0, 0)" in msg, msg


def _decode_step(G, cache, seed):
    ctxs = [700, 33, 1500, 2, 0, 900]
    D = 128
    qdt = "bf16"
    sp = wl.Spec("failure", len(ctxs), 2 * G, 2, D, 16, qdt, cache, 1.0 / math.sqrt(D),
                 np.array(ctxs, np.int32), spare_blocks=4, seed=seed)
    st = wl.structure(sp)
    hd = wl.host_data(sp, st)
    return GpuStep(sp, st, hd)


@pytest.mark.parametrize("cache", ["bf16", "e4m3"])
@pytest.mark.parametrize("G,part", [(1, 0), (2, 128), (4, 256), (8, 0), (2, 64)])
def test_decode_wait_that_runs_out(G, part, cache):
    g = _decode_step(G, cache, seed=50 + G)
    g.reshape()
    sp = g.sp
    _, _, ref = oracle_ref(g)
    cdt = pk.dtype_code(g.kc)
    ws = pk.decode_workspace(sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                             sp.block_size, g.max_ctx, part, cache_dtype=cdt)
    split = pk.decode_partition_tokens(sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                                       sp.block_size, g.max_ctx, part, cdt) < g.max_ctx
    g.out.fill_(float("nan"))
    pk.inject_wait_timeout(3, LIMIT_NS)        # tile 3 of (kv-head 0, sequence 0, part 0)
    pk.decode(g.out, g.q, g.kc, g.vc, g.bt, g.cl, g.max_ctx, sp.scale, k_scale=g.ks,
              v_scale=g.vs, partition_tokens=part, workspace=ws)
    # an E4M3 cache with head_dim 128 runs on the tcgen05 kernel (site 7)
    _expect_timeout(lambda: pk.decode_check(ws), 7 if cache == "e4m3" else 4)
    out = g.out_f64()
    assert np.isfinite(out).all()
    lost = np.zeros(out.shape[:2], bool)
    lost[0, :G] = True        # the rows of the unit that stopped: sequence 0, kv-head 0
    if not split:
        assert (out[lost] == 0).all()
    assert_close(out[~lost], ref[~lost], cache, "rows of the other units")
    # the same call again, without the injection: parity, and a clean check
    g.out.fill_(float("nan"))
    pk.decode(g.out, g.q, g.kc, g.vc, g.bt, g.cl, g.max_ctx, sp.scale, k_scale=g.ks,
              v_scale=g.vs, partition_tokens=part, workspace=ws)
    pk.decode_check(ws)
    assert_close(g.out_f64(), ref, cache, "clean call after the timeout")


def oracle_ref(g):
    from gpu_helpers import oracle_step
    return oracle_step(g.sp, g.st, g.hd)


def _prefill(ctxs, qlens, G, D, dt, seed, cache=None):
    sp = wl.Spec("failure", len(ctxs), 2 * G, 2, D, 16, dt, cache or dt, 1.0 / math.sqrt(D),
                 np.array(ctxs, np.int32), spare_blocks=3, seed=seed)
    st = wl.structure(sp)
    hd = wl.host_data(sp, st)
    qlens = np.array(qlens, np.int32)
    q = wl.prefill_queries_host(sp, qlens)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    ref = oracle.chunked_prefill(q, hd.key_cache, hd.value_cache, st.block_tables,
                                 sp.context_lens, cu, scale=np.float32(sp.scale),
                                 q_dtype=sp.q_dtype, cache_dtype=sp.cache_dtype,
                                 k_scale=hd.k_scale, v_scale=hd.v_scale)
    gq = dev(q, dt)
    kc, vc = dev(hd.key_cache, sp.cache_dtype), dev(hd.value_cache, sp.cache_dtype)
    ws = pk.chunked_prefill_workspace(sp.num_seqs, int(qlens.sum()), sp.num_heads,
                                      sp.num_kv_heads, D, int(qlens.max()), int(max(ctxs)),
                                      pk.dtype_code(kc))
    out = torch.full_like(gq, float("nan"))

    def call():
        pk.chunked_prefill(out, gq, i32(cu), int(qlens.max()), kc, vc, i32(st.block_tables),
                           i32(sp.context_lens), int(max(ctxs)), sp.scale,
                           k_scale=f32(hd.k_scale), v_scale=f32(hd.v_scale), workspace=ws)
    return sp, out, ws, call, ref


@pytest.mark.parametrize("kernel,cache,D,site", [
    ("mma_sync", "f16", 64, 5), ("mma_sync", "f16", 128, 5), ("mma_sync", "e4m3", 128, 5),
    ("tcgen05", "f16", 128, 6), ("tcgen05", "e4m3", 128, 6)])
def test_multi_token_wait_that_runs_out(kernel, cache, D, site):
    """mma.sync: 4-token chunks (4 rows per kv-head); tcgen05 rows on M: a
    128-token chunk, whose MMA warp must drain its MMAs before the tensor
    memory is freed."""
    G = 1
    if kernel == "tcgen05":
        ctxs, qlens = [300, 150, 128], [128, 100, 7]
    else:
        ctxs, qlens = [300, 90, 41], [4, 4, 2]
    dt = "bf16" if cache == "bf16" else "f16"
    sp, out, ws, call, ref = _prefill(ctxs, qlens, G, D, dt, seed=60 + site,
                                      cache=None if cache != "e4m3" else "e4m3")
    pk.inject_wait_timeout(5, LIMIT_NS)        # tile 5 of (sequence 0, kv-head 0, first tile)
    call()
    _expect_timeout(lambda: pk.decode_check(ws), site)
    o = out.double().cpu().numpy()
    assert np.isfinite(o).all()
    # rows of the first CTA: the first query tokens of sequence 0, heads of kv-head 0
    qt = {"mma_sync": 64 // G, "tcgen05": 128 // G}[kernel]
    lost = np.zeros(o.shape[:2], bool)
    lost[:min(qt, qlens[0]), :G] = True
    assert (o[lost] == 0).all()
    assert_close(o[~lost], ref[~lost], cache, "rows of the other CTAs")
    out.fill_(float("nan"))
    call()
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), ref, cache, "clean call after the timeout")


@pytest.mark.parametrize("cache", ["bf16", "e4m3"])
def test_short_chunks_on_tcgen05_wait_that_runs_out(cache):
    """Short chunks of many sequences run on tcgen05 with each of their at
    most 64 rows per unit held in two lanes, which take the two halves of
    every step and are merged at the end through shared memory behind a
    barrier of the softmax warps. A wait that runs out in the first unit must
    still let every softmax warp reach that barrier: the unit's rows are
    zeros, every other row matches the oracle, and the next call is clean."""
    G = 4
    rng = np.random.default_rng(81)
    n = 150  # x 2 kv-heads: 300 units, enough to fill the tcgen05 kernel's wave
    ctxs = rng.integers(100, 700, size=n)
    ctxs[0] = 600
    qlens = np.minimum(rng.integers(1, 9, size=n), ctxs)
    qlens[0] = 8
    sp, out, ws, call, ref = _prefill(list(ctxs), list(qlens), G, 128, "bf16", seed=83,
                                      cache=None if cache == "bf16" else "e4m3")
    pk.inject_wait_timeout(5, LIMIT_NS)  # tile 5 of sequence 0, kv-head 0
    call()
    _expect_timeout(lambda: pk.decode_check(ws), 6)
    o = out.double().cpu().numpy()
    assert np.isfinite(o).all()
    lost = np.zeros(o.shape[:2], bool)
    lost[:qlens[0], :G] = True  # the query tokens of sequence 0, heads of kv-head 0
    assert (o[lost] == 0).all()
    assert_close(o[~lost], ref[~lost], cache, "rows of the other units")
    out.fill_(float("nan"))
    call()
    pk.decode_check(ws)
    assert_close(out.double().cpu().numpy(), ref, cache, "clean call after the timeout")


def test_injection_is_used_up_and_can_be_cancelled():
    g = _decode_step(4, "bf16", seed=70)
    g.reshape()
    _, _, ref = oracle_ref(g)
    pk.inject_wait_timeout(2, LIMIT_NS)
    pk.inject_wait_timeout(-1, 0)               # cancelled: the next call is clean
    g.decode(partition_tokens=0)
    assert_close(g.out_f64(), ref, "bf16", "after a cancelled injection")
    with pytest.raises(pk.PagedError) as e:
        pk.inject_wait_timeout(1, 0)
    assert e.value.status == _native.PA_ERR_INVALID_ARG
