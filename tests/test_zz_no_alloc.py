"""pa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a serving loop that forbids cudaMalloc once running, a process
whose memory another framework's caching allocator already holds, a binding
without a device allocation API). It uses the library's own static device
scratch instead of a caller workspace.

Checked through the C ABI against the oracle, and against pa_decode (caller
workspace), on two calls in a row with different inputs; a call that needs
fewer partitions than the one before it, into a poisoned output, must use
only what it wrote itself; errors reach the caller through
pa_decode_noalloc_check; sizes beyond the static scratch are refused before
any launch. This file is collected last on purpose.
"""
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_448_b200 as pk
from paged_kv_cache_448_b200 import _native
from paged_kv_cache_448_b200 import workloads as wl
from gpu_helpers import GpuStep, assert_close, oracle_step

pytestmark = pytest.mark.gpu


def _noalloc(g, out, partition_tokens):
    sp = g.sp
    NB, BS, Hkv = g.kc.shape[:3]
    return _native.lib().pa_decode_noalloc(
        out.data_ptr(), g.q.data_ptr(), g.kc.data_ptr(), g.vc.data_ptr(), g.bt.data_ptr(),
        g.bt.shape[1], g.cl.data_ptr(), g.max_ctx, sp.num_seqs, sp.num_heads, Hkv,
        sp.head_dim, BS, NB, float(sp.scale), {"f16": 0, "bf16": 1}[sp.q_dtype],
        {"f16": 0, "bf16": 1, "e4m3": 2}[sp.cache_dtype],
        None if g.ks is None else g.ks.data_ptr(), None if g.vs is None else g.vs.data_ptr(),
        partition_tokens, torch.cuda.current_stream().cuda_stream)


def _check():
    return _native.lib().pa_decode_noalloc_check(torch.cuda.current_stream().cuda_stream)


def _workload(ctxs, H, Hkv, D, bs, qdt, cdt, seed):
    sp = wl.Spec("noalloc", len(ctxs), H, Hkv, D, bs, qdt, cdt, 1.0 / math.sqrt(D),
                 np.array(ctxs, np.int32), spare_blocks=5, seed=seed)
    st = wl.structure(sp)
    return GpuStep(sp, st, wl.host_data(sp, st))


def test_noalloc_matches_oracle_and_decode_on_two_calls_in_a_row():
    # two different batches, both on the partitioned path (scratch in use)
    steps = [(_workload([700, 33, 1500, 2, 0, 900], 16, 4, 128, 16, "bf16", "bf16", 1), 256),
             (_workload([1200, 400, 64, 2047], 8, 8, 64, 32, "f16", "f16", 2), 128)]
    assert _check() == _native.PA_OK, _native.lib().pa_last_error()
    for g, part in steps:
        g.reshape()
        _, _, ref = oracle_step(g.sp, g.st, g.hd)
        g.decode(partition_tokens=part)                   # existing entry point
        expect = g.out_f64().copy()
        out = torch.full_like(g.q, float("nan"))
        assert _noalloc(g, out, part) == _native.PA_OK, _native.lib().pa_last_error()
        assert _check() == _native.PA_OK, _native.lib().pa_last_error()
        got = out.double().cpu().numpy()
        assert_close(got, ref, g.sp.cache_dtype, "noalloc vs oracle")
        assert_close(got, expect, g.sp.cache_dtype, "noalloc vs decode")


def test_noalloc_fewer_partitions_after_a_larger_call():
    """Call 1 fills the scratch with the partials of a large batch (many
    partitions per row); call 2 needs fewer partitions per row and writes
    into a poisoned output: its combine may only read what it wrote."""
    big = _workload([4000, 3900, 2500, 4096, 3000, 1000, 4000, 2222], 32, 8, 128, 16, "f16",
                    "f16", 5)
    big.reshape()
    out = torch.zeros_like(big.q)
    assert _noalloc(big, out, 128) == _native.PA_OK, _native.lib().pa_last_error()
    small = _workload([300, 1, 257, 512], 16, 4, 128, 16, "f16", "f16", 6)
    small.reshape()
    _, _, ref = oracle_step(small.sp, small.st, small.hd)
    out = torch.full_like(small.q, float("nan"))
    assert _noalloc(small, out, 256) == _native.PA_OK, _native.lib().pa_last_error()
    assert _check() == _native.PA_OK, _native.lib().pa_last_error()
    assert_close(out.double().cpu().numpy(), ref, "f16", "fewer partitions after a big call")


def test_noalloc_check_reports_errors():
    g = _workload([700, 33, 900], 8, 2, 128, 16, "bf16", "bf16", 7)
    g.reshape()
    out = torch.zeros_like(g.q)
    # a block id outside the pool: read as zeros and reported as a table error
    good = g.bt.clone()
    g.bt[1, 0] = g.kc.shape[0] + 3
    assert _noalloc(g, out, 256) == _native.PA_OK
    assert _check() == _native.PA_ERR_BAD_TABLE
    assert b"outside the pool" in _native.lib().pa_last_error()
    assert _check() == _native.PA_OK                       # read and cleared
    g.bt.copy_(good)
    # a pipeline wait that runs out (tile 2 of the first unit left out)
    pk.inject_wait_timeout(2, 20_000_000)
    assert _noalloc(g, out, 256) == _native.PA_OK
    assert _check() == _native.PA_ERR_CUDA
    assert b"timed out" in _native.lib().pa_last_error()
    # and the next call is clean again
    _, _, ref = oracle_step(g.sp, g.st, g.hd)
    assert _noalloc(g, out, 256) == _native.PA_OK
    assert _check() == _native.PA_OK
    assert_close(out.double().cpu().numpy(), ref, "bf16", "after the reported errors")


def test_noalloc_refuses_sizes_beyond_its_scratch():
    g = _workload([64], 8, 8, 128, 16, "f16", "f16", 3)
    out = torch.zeros_like(g.q)
    # 4096 sequences x 8 heads x 1024 partitions of 16 tokens would need GBs
    lib = _native.lib()
    st = lib.pa_decode_noalloc(out.data_ptr(), g.q.data_ptr(), g.kc.data_ptr(), g.vc.data_ptr(),
                               g.bt.data_ptr(), g.bt.shape[1], g.cl.data_ptr(), 16384, 4096, 8,
                               8, 128, 16, g.kc.shape[0], 0.1, 0, 0, None, None, 16,
                               torch.cuda.current_stream().cuda_stream)
    assert st == _native.PA_ERR_UNSUPPORTED
    assert b"static scratch" in lib.pa_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0                 # nothing was launched
