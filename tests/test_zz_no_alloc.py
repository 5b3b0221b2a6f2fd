"""pa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a serving loop that forbids cudaMalloc once running, a process
whose memory another framework's caching allocator already holds, a binding
without a device allocation API). It uses the library's own static device
scratch instead of a caller workspace.

Checked through the C ABI against pa_decode (caller workspace) on two calls in
a row with different inputs, so a second call cannot pass by reusing what the
first left in the shared scratch; sizes beyond the static scratch are refused
before any launch. This file is collected last on purpose.
"""
import math

import numpy as np
import pytest
import torch

from paged_kv_cache_448_b200 import _native
from paged_kv_cache_448_b200 import workloads as wl
from gpu_helpers import GpuStep, assert_close

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


def _workload(ctxs, H, Hkv, D, bs, qdt, cdt, seed):
    sp = wl.Spec("noalloc", len(ctxs), H, Hkv, D, bs, qdt, cdt, 1.0 / math.sqrt(D),
                 np.array(ctxs, np.int32), spare_blocks=5, seed=seed)
    st = wl.structure(sp)
    return GpuStep(sp, st, wl.host_data(sp, st))


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    # two different batches, both on the partitioned path (scratch in use)
    steps = [(_workload([700, 33, 1500, 2, 0, 900], 16, 4, 128, 16, "bf16", "bf16", 1), 256),
             (_workload([1200, 400, 64, 2047], 8, 8, 64, 32, "f16", "f16", 2), 128)]
    for g, part in steps:
        g.reshape()
        g.decode(partition_tokens=part)                   # existing entry point
        expect = g.out_f64().copy()
        out = torch.full_like(g.q, float("nan"))
        assert _noalloc(g, out, part) == _native.PA_OK, _native.lib().pa_last_error()
        torch.cuda.synchronize()
        assert_close(out.double().cpu().numpy(), expect, g.sp.cache_dtype, "noalloc vs decode")


def test_noalloc_refuses_sizes_beyond_its_scratch():
    g = _workload([64], 8, 8, 128, 16, "f16", "f16", 3)
    out = torch.zeros_like(g.q)
    # 65535 sequences x 8 heads x 1024 partitions of 16 tokens would need GBs
    lib = _native.lib()
    st = lib.pa_decode_noalloc(out.data_ptr(), g.q.data_ptr(), g.kc.data_ptr(), g.vc.data_ptr(),
                               g.bt.data_ptr(), g.bt.shape[1], g.cl.data_ptr(), 16384, 4096, 8,
                               8, 128, 16, g.kc.shape[0], 0.1, 0, 0, None, None, 16,
                               torch.cuda.current_stream().cuda_stream)
    assert st == _native.PA_ERR_UNSUPPORTED
    assert b"static scratch" in lib.pa_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0                 # nothing was launched
