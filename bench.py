#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

One step = one decode step of a LLaMA-7B-shaped layer (32 sequences x 2048
context tokens, 32 heads, head_dim 128, block_size 16, fp16 K/V, pool of
32*128+256 shuffled blocks): reshape_and_cache of the step's 32 new tokens
into their slots, then paged decode attention over the whole context.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU. Under a launcher (torch.distributed.run sets
WORLD_SIZE) each process is one rank; `--gpus N` started as a plain process
starts the N ranks itself through torch.distributed.run. Every rank runs its
own batch on its own GPU (sequences are independent; no collective on the
data path, NCCL only for the barrier and the maximum of the times): weak
scaling, value = bytes of all ranks / max-over-ranks device time.

Rank 0 prints one JSON line. `value` is KV-read GB/s: the decode's
algorithmic bytes (K/V rows read once per kv-head + query + output + block
table entries + context lengths) per step over the device time of the step.
`--impl reference` times the CPU oracle (plain fp64 C) on the host cores
instead, on a sample of the same workload sized so the run ends in minutes.

The other rows of the path, one JSON line each (a default run at one GPU
also measures each of them, with fewer steps, in a child process of its own
after the headline, and adds a summary of each under the line's "rows" key;
--no-rows leaves them out):
    --op prefill --workload chunk_llama7b|chunk_gqa70b|verify_gqa70b|chunk_gqa70b_fp8
        multi-token query (TFLOP/s; against the tensor or HBM roofline,
        whichever the work per byte makes binding)
    --op copy_blocks    copy-on-write copies of 2048 blocks (GB/s read + write)
    --op swap           512 blocks to a pinned host pool and back (GB/s)
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_448_b200 import workloads as wl  # noqa: E402

METRIC = "paged-decode KV-read GB/s (% of B200 HBM peak); decode tokens/s per layer"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=2, help="workload 1..5 (2 = headline)")
    ap.add_argument("--partition", type=int, default=-1,
                    help="decode partition tokens (-1: the workload's setting, 0: automatic)")
    ap.add_argument("--op", choices=["decode", "prefill", "copy_blocks", "swap"],
                    default="decode",
                    help="decode: the headline step; the others time the multi-token query "
                         "path or the block-copy kernel on their own workloads")
    ap.add_argument("--workload", default="chunk_llama7b",
                    help="multi-token workload for --op prefill: " + ", ".join(wl.PREFILL_NAMES))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-rows", action="store_true",
                    help="leave out the other rows of the path (measured by default with "
                         "the headline at one GPU, under the line's \"rows\" key)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor TFLOP/s (burst: a kernel timed alone)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


# The units each bench row's kernels are built from (plus everything they
# include, and api.cu, which launches them).
OP_UNITS = {"decode": ("decode_*.cu",), "prefill": ("prefill_*.cu",),
            "copy_blocks": ("copy_blocks.cu",)}


def op_sources(op: str = "decode") -> list:
    """The files the kernels of a bench row are built from: its units,
    everything they include (transitively), and api.cu."""
    import re
    csrc = os.path.join(ROOT, "paged_kv_cache_448_b200", "csrc")
    todo = [os.path.join(csrc, "api.cu")]
    for pat in OP_UNITS[op]:
        todo += sorted(glob.glob(os.path.join(csrc, pat)))
    seen = set()
    while todo:
        f = todo.pop()
        if f in seen or not os.path.exists(f):
            continue
        seen.add(f)
        with open(f, encoding="utf-8") as fh:
            for inc in re.findall(r'^#include "([^"]+)"', fh.read(), re.M):
                todo.append(os.path.join(csrc, inc))
    return sorted(seen)


def decode_sources() -> list:
    return op_sources("decode")


def sources_digest(op: str = "decode") -> str:
    """Digest of a row's kernel sources: a recorded DRAM traffic figure stands
    only for the exact sources it was taken on."""
    h = hashlib.sha256()
    for f in op_sources(op):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(workload: str, op: str = "decode"):
    """DRAM bytes (read + write) per launch of a row's dominant kernel from the
    committed ncu record, if it was taken on the current sources of that row
    and on this workload; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        entries = json.load(f).get("entries", [])
    for e in entries:
        if e.get("op") == op and e.get("workload") == workload and \
                e.get("sources_sha256") == sources_digest(op):
            return e.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception as e:  # no nvidia-smi: clocks unknown
            log("clock sampler unavailable:", e)
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) != len(self.FIELDS):
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def workload_name(sp: wl.Spec, st: wl.Structure) -> str:
    ctx = sp.context_lens
    ctxs = f"ctx {int(ctx[0])}" if ctx.min() == ctx.max() else f"ctx {int(ctx.min())}-{int(ctx.max())}"
    return (f"{sp.name}: {sp.num_seqs} seqs, {ctxs}, {sp.num_heads} q / {sp.num_kv_heads} kv heads, "
            f"head_dim {sp.head_dim}, block_size {sp.block_size}, q {sp.q_dtype}, "
            f"KV {sp.cache_dtype}, pool {st.num_blocks} shuffled blocks")


# ------------------------------------------------------------------ CPU oracle

def oracle_sample(sp: wl.Spec, seqs: int, heads: int):
    """A sub-workload of the same shape (first `seqs` sequences, `heads` kv-heads
    and their query groups) with its host inputs, for timing the oracle."""
    g = sp.num_heads // sp.num_kv_heads
    # shared prefixes become private copies: the oracle gathers each
    # sequence's contiguous K/V either way
    sub = dataclasses.replace(sp, num_seqs=seqs, context_lens=sp.context_lens[:seqs].copy(),
                              num_kv_heads=heads, num_heads=heads * g, spare_blocks=0,
                              shared_groups=0, prefix_tokens=0)
    st = wl.structure(sub)
    return sub, st, wl.host_data(sub, st)


def time_oracle(sub, st, hd) -> float:
    import oracle
    t0 = time.perf_counter()
    oracle.decode(hd.query, hd.key_cache, hd.value_cache, st.block_tables, sub.context_lens,
                  scale=np.float32(sub.scale), q_dtype=sub.q_dtype, cache_dtype=sub.cache_dtype,
                  k_scale=hd.k_scale, v_scale=hd.v_scale)
    return time.perf_counter() - t0


def _oracle_worker(sp, seq_ids, barrier, results):
    """Process of the all-cores timing: builds the inputs of its sequences
    (each alone: all heads, full context), waits for every process, then
    times the oracle on them; reports (bytes, start, end) by wall clock."""
    import oracle
    oracle.build()
    jobs = []
    for i in seq_ids:
        sub = dataclasses.replace(sp, num_seqs=1, context_lens=sp.context_lens[i:i + 1].copy(),
                                  spare_blocks=0, shared_groups=0, prefix_tokens=0)
        st = wl.structure(sub)
        jobs.append((sub, st, wl.host_data(sub, st)))
    barrier.wait(timeout=120)
    t0 = time.time()
    nbytes = 0
    for sub, st, hd in jobs:
        time_oracle(sub, st, hd)
        nbytes += wl.decode_bytes(sub, st)
    results.put((nbytes, t0, time.time()))


def cpu_baseline_all_cores(sp: wl.Spec, t_seq: float, budget_s: float) -> dict:
    """The same oracle on every host core at once: one process per core
    (started with spawn, as the GPU is already in use here), sequences dealt
    round-robin; inputs are built before a barrier, and the time is from the
    first process's start to the last one's end."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    workers = max(1, min(os.cpu_count() or 1, 64, sp.num_seqs))
    rounds = max(1, int(budget_s // max(t_seq, 1e-3)))
    seqs = min(sp.num_seqs, workers * rounds)
    barrier, results = ctx.Barrier(workers), ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker,
                         args=(sp, list(range(w, seqs, workers)), barrier, results))
             for w in range(workers)]
    for p in procs:
        p.start()
    try:
        res = [results.get(timeout=120 + 4 * budget_s) for _ in procs]
    finally:
        for p in procs:  # the processes started above, and no others
            p.join(timeout=5)
            if p.is_alive():
                p.terminate()
                p.join(timeout=5)
    t = max(r[2] for r in res) - min(r[1] for r in res)
    gb = sum(r[0] for r in res) / 1e9
    return {"value": round(gb / t, 4), "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": f"first {seqs} of {sp.num_seqs} sequences dealt over {workers} "
                      f"processes; {t:.1f} s wall",
            "tokens_per_s_per_layer": round(seqs / t, 3)}


def cpu_baseline(sp: wl.Spec, budget_s: float) -> dict:
    """The oracle as it stands (single-threaded C, fp64) on a bounded sample,
    and the same oracle on all host cores (`all_cores`)."""
    import oracle
    oracle.build()
    one = oracle_sample(sp, 1, sp.num_kv_heads)
    t1 = time_oracle(*one)
    seqs = int(max(1, min(sp.num_seqs, budget_s // max(t1, 1e-3))))
    sub = oracle_sample(sp, seqs, sp.num_kv_heads)
    t = time_oracle(*sub)
    gb = wl.decode_bytes(sub[0], sub[1]) / 1e9
    out = {"value": round(gb / t, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"first {seqs} of {sp.num_seqs} sequences of the same workload "
                     f"(all {sp.num_heads} heads, full contexts); {t:.1f} s single-threaded fp64 C",
           "tokens_per_s_per_layer": round(seqs / t, 3)}
    try:
        out["all_cores"] = cpu_baseline_all_cores(sp, t1, budget_s)
    except Exception as e:  # the single-threaded figure stands on its own
        out["all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"}
    return out


def run_reference(args, sp, st):
    """--impl reference: the oracle on the host cores, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    budget = 12.5 * args.cpu_seconds    # 150 s of oracle work at the default 12
    per_step = budget / max(1, args.steps + args.warmup)
    one_head = oracle_sample(sp, 1, 1)
    t_pair = time_oracle(*one_head)
    pairs_total = sp.num_seqs * sp.num_kv_heads
    pairs = int(max(1, min(pairs_total, per_step // max(t_pair, 1e-4))))
    if pairs >= sp.num_kv_heads:
        seqs, heads = max(1, pairs // sp.num_kv_heads), sp.num_kv_heads
    else:
        seqs, heads = 1, pairs
    sub = oracle_sample(sp, seqs, heads)
    for _ in range(args.warmup):
        time_oracle(*sub)
    t = sum(time_oracle(*sub) for _ in range(args.steps))
    gb = wl.decode_bytes(sub[0], sub[1]) / 1e9 * args.steps
    value = gb / t
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(sp, st), "global_batch": sp.num_seqs,
                       "seq_len": int(sp.context_lens.max()), "parallelism": "none (host CPU)"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1,
                             "kind": "oracle",
                             "sample": f"each step: {seqs} sequence(s) x {heads} kv-head(s) of "
                                       f"the workload, full context, single-threaded fp64 C"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- rank logic

def rank_seed(sp: wl.Spec, rank: int) -> int:
    """Each rank decodes its own batch of the same shape (weak scaling)."""
    return sp.seed + 97 * rank


def max_over_ranks(values, world: int, device):
    """Element-wise maximum over all ranks (the slowest rank sets the time)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput_gbs(world: int, bytes_per_rank: int, ms: float) -> float:
    """Whole-job GB/s: the bytes all ranks processed over the slowest rank's time."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


# ------------------------------------------------------------------ GPU arm

# ------------------------------------------------ other rows of the hot path

def _time_device(fn, steps, warmup):
    """Mean ms per call over `steps` calls (CUDA events on the current stream)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def prefill_oracle_sample(sp, qlens, budget_s):
    """Oracle timing on the first sequences of the multi-token workload (all
    heads, full contexts), as many as fit about `budget_s` seconds."""
    import oracle
    oracle.build()
    done, t_total, flops = 0, 0.0, 0
    while done < sp.num_seqs and t_total < budget_s:
        sub = dataclasses.replace(sp, num_seqs=1, context_lens=sp.context_lens[done:done + 1].copy(),
                                  spare_blocks=0)
        st = wl.structure(sub)
        hd = wl.host_data(sub, st)
        ql = qlens[done:done + 1]
        q = wl.prefill_queries_host(sub, ql)
        t0 = time.perf_counter()
        oracle.chunked_prefill(q, hd.key_cache, hd.value_cache, st.block_tables, sub.context_lens,
                               np.array([0, ql[0]], np.int32), scale=np.float32(sp.scale),
                               q_dtype=sp.q_dtype, cache_dtype=sp.cache_dtype,
                               k_scale=hd.k_scale, v_scale=hd.v_scale)
        t_total += time.perf_counter() - t0
        flops += wl.prefill_flops(sub, ql)
        done += 1
    return {"value": round(flops / t_total / 1e12, 6), "unit": "TFLOP/s", "cores": 1,
            "kind": "oracle",
            "sample": f"first {done} of {sp.num_seqs} sequences (all heads, whole chunks); "
                      f"{t_total:.1f} s single-threaded fp64 C"}


def run_prefill(args):
    """--op prefill: the multi-token query path on one multi-token workload."""
    import torch
    import paged_kv_cache_448_b200 as pk
    sp, qlens = wl.prefill_spec(args.workload)
    flops, nbytes = wl.prefill_flops(sp, qlens), wl.prefill_bytes(sp, qlens)
    chunk = int(qlens.max())
    config = {"workload": f"{sp.name}: {sp.num_seqs} seqs x {chunk} query tokens, ctx "
                          f"{int(sp.context_lens.min())}-{int(sp.context_lens.max())}, "
                          f"{sp.num_heads} q / {sp.num_kv_heads} kv heads, head_dim {sp.head_dim}, "
                          f"block_size {sp.block_size}, {sp.q_dtype} query, "
                          f"{sp.cache_dtype} cache"}
    # tensor-bound when the work per K/V byte is above the machine balance
    peak_t, kind_t = measured_tensor_peak()
    kind_t = f"{kind_t} dense bf16 (cuBLAS)"
    G = sp.num_heads // sp.num_kv_heads
    if sp.cache_dtype == "e4m3" and sp.head_dim == 128 and chunk * G >= 128:
        # the tcgen05 kernel runs 8-bit MMAs (kind::f8f6f4): nominal fp8 = 2 x bf16
        peak_t, kind_t = round(2 * peak_t, 1), f"{kind_t} x 2 (nominal fp8 / bf16 ratio)"
    peak_b, kind_b = measured_peaks()
    tensor_bound = flops / nbytes > peak_t * 1e12 / (peak_b * 1e9)
    if args.impl == "reference":
        cb = prefill_oracle_sample(sp, qlens, args.cpu_seconds)
        print(json.dumps({"metric": "multi-token paged attention TFLOP/s", "impl": "reference",
                          "value": cb["value"], "unit": "TFLOP/s", "n_gpus": 1,
                          "higher_is_better": True, "config": config, "cpu_baseline": cb,
                          "e2e": {"value": cb["value"], "unit": "TFLOP/s",
                                  "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return
    dev = torch.device("cuda", 0)
    st = wl.structure(sp)
    d = wl.device_data(sp, st, device=dev)
    q = wl.prefill_queries_device(sp, qlens, device=dev)
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)).to(dev)
    bt = torch.from_numpy(st.block_tables).to(dev)
    cl = torch.from_numpy(sp.context_lens).to(dev)
    out = torch.empty_like(q)
    ws = pk.chunked_prefill_workspace(sp.num_seqs, int(qlens.sum()), sp.num_heads,
                                      sp.num_kv_heads, sp.head_dim, chunk,
                                      int(sp.context_lens.max()),
                                      pk.dtype_code(d["key_cache"]), device=dev)
    mctx = int(sp.context_lens.max())
    fn = lambda: pk.chunked_prefill(out, q, cu, chunk, d["key_cache"], d["value_cache"], bt, cl,
                                    mctx, sp.scale, k_scale=d["k_scale"], v_scale=d["v_scale"],
                                    workspace=ws)
    sampler = ClockSampler(0)
    sampler.start()
    ms = _time_device(fn, args.steps, max(3, args.warmup))
    clocks = sampler.stop()
    pk.decode_check(ws)
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    roof = ({"bound": "tensor", "achieved": round(tflops, 2), "peak": peak_t, "unit": "TFLOP/s",
             "frac": round(tflops / peak_t, 4), "peak_kind": kind_t}
            if tensor_bound else
            {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak_b, "unit": "GB/s",
             "frac": round(gbs / peak_b, 4), "peak_kind": f"{kind_b} HBM copy GB/s"})
    roof.update({"traffic": recorded_traffic(sp.name, "prefill"),
                 "algorithmic_flops_per_launch": flops,
                 "algorithmic_bytes_per_launch": nbytes, "launch_ms": round(ms, 5)})
    line = {"metric": "multi-token paged attention TFLOP/s", "value": round(tflops, 3),
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": sp.q_dtype, "data": "synthetic", "config": config,
            "gb_per_s": round(gbs, 2),
            "query_tokens_per_s": round(int(qlens.sum()) / (ms * 1e-3), 1),
            "roofline": roof, "gpu_launches": args.steps, "clocks": clocks}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = prefill_oracle_sample(sp, qlens, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_copy(args):
    """--op copy_blocks: copy-on-write copies of 2048 random block pairs inside
    the LLaMA-7B-shaped cache (K and V); --op swap: 512 of its blocks out to a
    pinned host pool and back in."""
    import torch
    import paged_kv_cache_448_b200 as pk
    dev = torch.device("cuda", 0)
    NB, BS, H, D = 4352, 16, 32, 128
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    k = torch.randn((NB, BS, H, D), generator=g, device=dev, dtype=torch.float32).half()
    v = torch.randn((NB, BS, H, D), generator=g, device=dev, dtype=torch.float32).half()
    bb = BS * H * D * 2
    rng = np.random.default_rng(1234)
    perm = rng.permutation(NB)
    sampler = ClockSampler(0)
    if args.op == "copy_blocks":
        n = 2048
        pairs = torch.from_numpy(np.stack([perm[:n], perm[n:2 * n]], 1).astype(np.int32)).to(dev)
        sampler.start()
        ms = _time_device(lambda: pk.copy_blocks(k, v, k, v, pairs), args.steps,
                          max(3, args.warmup))
        clocks = sampler.stop()
        moved = 2 * 2 * n * bb                                     # read + write, K and V
        peak, kind = measured_peaks()
        gbs = moved / (ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak, "unit": "GB/s",
                "frac": round(gbs / peak, 4), "peak_kind": f"{kind} HBM copy GB/s",
                "traffic": recorded_traffic("copy_blocks", "copy_blocks"),
                "algorithmic_bytes_per_launch": moved, "launch_ms": round(ms, 5)}
        metric, workload = "block copy GB/s (read + write)", \
            f"copy-on-write: {n} block pairs of a 4352-block fp16 cache (16 x 32 x 128), K and V"
    else:
        n = 512
        hk = torch.empty((n, BS, H, D), dtype=torch.float16).pin_memory()
        hv = torch.empty_like(hk).pin_memory()
        out_p = torch.from_numpy(np.stack([perm[:n], np.arange(n)], 1).astype(np.int32)).to(dev)
        in_p = torch.from_numpy(np.stack([np.arange(n), perm[n:2 * n]], 1).astype(np.int32)).to(dev)
        sampler.start()
        ms = _time_device(lambda: (pk.copy_blocks(k, v, hk, hv, out_p),
                                   pk.copy_blocks(hk, hv, k, v, in_p)), args.steps,
                          max(3, args.warmup))
        clocks = sampler.stop()
        big = torch.empty(n * bb, dtype=torch.uint8).pin_memory()
        dbig = torch.empty(n * bb, dtype=torch.uint8, device=dev)
        ref_ms = _time_device(lambda: (dbig.copy_(big, non_blocking=True),
                                       big.copy_(dbig, non_blocking=True)), 5, 2)
        moved = 2 * 2 * n * bb                                     # out and in, K and V
        peak = round(2 * n * bb / (ref_ms * 1e-3) / 1e9, 2)
        gbs = moved / (ms * 1e-3) / 1e9
        roof = {"bound": "pcie", "achieved": round(gbs, 2), "peak": peak, "unit": "GB/s",
                "frac": round(gbs / peak, 4),
                "peak_kind": "measured in this run: contiguous pinned cudaMemcpy, one H2D + one D2H",
                "traffic": None, "algorithmic_bytes_per_launch": moved, "launch_ms": round(ms, 5)}
        metric, workload = "block swap GB/s (GPU <-> pinned host)", \
            f"swap: {n} blocks of a 4352-block fp16 cache (16 x 32 x 128) out to pinned host and back, K and V"
    print(json.dumps({"metric": metric, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": 1,
                      "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                      "dtype": "f16", "data": "synthetic", "config": {"workload": workload},
                      "roofline": roof, "gpu_launches": args.steps * (1 if args.op == "copy_blocks" else 2),
                      "clocks": clocks}), flush=True)


# The other rows of the hot path: (name, arguments of this script). A default
# run at one GPU measures each in a child process of its own after the
# headline, with fewer steps, and reports a summary under "rows".
ROWS = [
    ("llama13b_mix", ["--config", "3", "--no-e2e"]),
    ("gqa70b_long", ["--config", "4", "--no-e2e"]),
    ("prefix_fp8", ["--config", "5", "--no-e2e"]),
    ("chunk_llama7b", ["--op", "prefill", "--workload", "chunk_llama7b"]),
    ("chunk_gqa70b", ["--op", "prefill", "--workload", "chunk_gqa70b"]),
    ("verify_gqa70b", ["--op", "prefill", "--workload", "verify_gqa70b"]),
    ("chunk_gqa70b_fp8", ["--op", "prefill", "--workload", "chunk_gqa70b_fp8"]),
    ("copy_blocks", ["--op", "copy_blocks"]),
    ("swap", ["--op", "swap"]),
]
ROW_STEPS, ROW_WARMUP = 500, 5


def row_summary(name: str, line: dict) -> dict:
    """The figures of a row's JSON line that the headline line carries."""
    out = {"row": name}
    for k in ("metric", "value", "unit", "ms_per_step", "dtype"):
        if k in line:
            out[k] = line[k]
    roof = line.get("roofline") or {}
    out["roofline"] = {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                            "traffic", "peak_kind") if k in roof}
    clocks = line.get("clocks") or {}
    out["clocks"] = {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons") if k in clocks}
    return out


def run_rows(rows=None, budget_s: float = 300.0, child_timeout_s: float = 150.0,
             command=None) -> list:
    """Each row measured by this script in a child process, one after the
    other, so that a row's failure, hang or memory cannot reach the headline's
    measurement or line: a row that fails or runs out of time is reported as
    such. `command(args)` builds a child's command line."""
    rows = ROWS if rows is None else rows
    if command is None:
        def command(extra):
            return ([sys.executable, os.path.abspath(__file__), "--steps", str(ROW_STEPS),
                     "--warmup", str(ROW_WARMUP), "--no-cpu-baseline", "--no-rows"] + extra)
    out = []
    t_end = time.time() + budget_s
    for name, extra in rows:
        left = t_end - time.time()
        if left < 10:
            out.append({"row": name, "skipped": "the time budget of the rows was spent"})
            continue
        try:
            r = subprocess.run(command(extra), capture_output=True, text=True, cwd=ROOT,
                               timeout=min(child_timeout_s, left))
        except subprocess.TimeoutExpired:
            out.append({"row": name, "error": "timed out"})
            continue
        lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
        if r.returncode != 0 or not lines:
            tail = (r.stderr.strip().splitlines() or ["no output"])[-1][:200]
            out.append({"row": name, "error": f"exit {r.returncode}: {tail}"})
            continue
        try:
            out.append(row_summary(name, json.loads(lines[-1])))
        except ValueError as e:
            out.append({"row": name, "error": f"unreadable line: {e}"})
    return out


def relaunch_command(gpus: int, port: int, argv: list) -> list:
    """One process per GPU through torch.distributed.run on this node (the
    form the multi-GPU contract uses), bounded by `timeout` as the last
    resort; the process group itself has a short timeout."""
    return ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run",
            "--nnodes=1", f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1",
            f"--master-port={port}", os.path.abspath(__file__)] + list(argv)


def relaunch(args) -> int:
    """`--gpus N` (N > 1) started as a plain process: start N ranks and pass
    rank 0's line through."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    return subprocess.call(relaunch_command(args.gpus, port, sys.argv[1:]))


def world_of(args) -> tuple:
    """(world, rank, local rank) from the launcher's environment; the world
    must be the --gpus the run was asked for."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but {world} rank(s) were started")
    return world, rank, local


def decode_line(args, sp: wl.Spec, st: wl.Structure, world: int, step_ms: float,
                dec_ms: float, eff_part: int, launches_per_step: int, clocks: dict,
                e2e=None) -> dict:
    """The JSON line of a decode run from the max-over-ranks times: `value`
    is every rank's bytes over the slowest rank's step time."""
    dbytes = wl.decode_bytes(sp, st)
    max_ctx = int(sp.context_lens.max())
    split = eff_part < max_ctx
    peak, peak_kind = measured_peaks()
    value = job_throughput_gbs(world, dbytes, step_ms)
    achieved = dbytes / (dec_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": sp.cache_dtype, "data": "synthetic",
        "config": {"workload": workload_name(sp, st), "global_batch": sp.num_seqs * world,
                   "seq_len": max_ctx, "parallelism": f"dp{world}",
                   "partition_tokens": eff_part if split else None,
                   "l2": f"inputs larger than L2: {wl.kv_bytes(sp) / 1e9:.2f} GB of K/V "
                         "per step vs 126 MB L2; no flush"},
        "pct_of_nominal_8000": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        # against the copy bandwidth measured on this machine, or the fallback
        # figure when no measurement is present (peak_kind says which)
        "pct_of_copy_peak": round(100 * value / world / peak, 2),
        "tokens_per_s_per_layer": round(world * sp.num_seqs / (step_ms * 1e-3), 1),
        "roofline": {"bound": "hbm", "kernel": "pa_decode (decode" +
                     (" + partition combine)" if split else ")"),
                     "achieved": round(achieved, 2), "peak": peak,
                     "peak_kind": f"{peak_kind} HBM copy GB/s", "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic(sp.name, "decode"),
                     "algorithmic_bytes_per_launch": dbytes,
                     "launch_ms": round(dec_ms, 5)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if e2e:
        line["e2e"] = {"value": round(job_throughput_gbs(world, dbytes, e2e["ms_per_step"]), 2),
                       "unit": "GB/s", "h2d_bytes_per_step": e2e["h2d"],
                       "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": round(e2e["ms_per_step"], 5),
                       "copies": "one packed host-to-device copy of the step's inputs and one "
                                 "device-to-host copy of its output per step, on an upload and a "
                                 "read-back stream, double-buffered so they overlap the "
                                 "neighbouring steps",
                       "checked": "both read-back buffers equal the device-timed loop's "
                                  "output bit for bit"}
    return line


class E2EStep:
    """One decode step through the public API from pinned host memory: the
    step's inputs (query, new K/V, block table, context lengths, slots) are
    packed in one pinned buffer and uploaded by one copy, and the output is
    read back by one copy, on an upload stream and a read-back stream. Two
    device buffers of each alternate, so the upload of step k+1 and the
    read-back of step k-1 run under the decode of step k."""

    NAMES = ("query", "new_key", "new_value", "bt", "cl", "sl")

    def __init__(self, host: dict, out_like, run_step, device):
        import torch
        offs, at = {}, 0
        for k in self.NAMES:
            offs[k] = at
            at = (at + host[k].numel() * host[k].element_size() + 255) // 256 * 256
        self.nbytes = at
        self.pin_in = torch.empty(at, dtype=torch.uint8).pin_memory()
        for k in self.NAMES:
            t = host[k].contiguous().view(-1).view(torch.uint8)
            self.pin_in[offs[k]:offs[k] + t.numel()].copy_(t)
        self.h2d = sum(host[k].numel() * host[k].element_size() for k in self.NAMES)
        self.dev_in = [torch.empty(at, dtype=torch.uint8, device=device) for _ in range(2)]
        self.views = []
        for b in range(2):
            v = {}
            for k in self.NAMES:
                n = host[k].numel() * host[k].element_size()
                v[k] = self.dev_in[b][offs[k]:offs[k] + n].view(host[k].dtype).view(host[k].shape)
            self.views.append(v)
        self.out = [torch.empty_like(out_like) for _ in range(2)]
        self.pin_out = [torch.empty(out_like.shape, dtype=out_like.dtype).pin_memory()
                        for _ in range(2)]
        self.d2h = out_like.numel() * out_like.element_size()
        # uploads and read-backs on streams of their own: a read-back waits for
        # its step's decode, and the next upload must not queue behind it
        self.up = torch.cuda.Stream(device=device)
        self.down = torch.cuda.Stream(device=device)
        self.compute = torch.cuda.current_stream(device)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        self.uploaded, self.done, self.read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        self.run_step = run_step
        # the same per-step event pair around the decode as in the device-timed
        # loop, so that both loops carry the same instrumentation
        self.ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        self.k = 0
        for b in range(2):  # every buffer starts free
            self.done[b].record(self.compute)
            self.read[b].record(self.down)

    def __call__(self):
        import torch
        b = self.k & 1
        with torch.cuda.stream(self.up):
            # buffer pair b is free once the decode of step k-2 read its inputs
            # and that step's output was read back; the upload stream takes
            # both waits, so the decode waits for the upload alone
            self.up.wait_event(self.done[b])
            self.up.wait_event(self.read[b])
            self.dev_in[b].copy_(self.pin_in, non_blocking=True)
            self.uploaded[b].record(self.up)
        self.compute.wait_event(self.uploaded[b])
        v = self.views[b]
        self.run_step(v["query"], v["new_key"], v["new_value"], v["bt"], v["cl"], v["sl"],
                      self.out[b], self.ev)
        self.done[b].record(self.compute)
        with torch.cuda.stream(self.down):
            self.down.wait_event(self.done[b])
            self.pin_out[b].copy_(self.out[b], non_blocking=True)
            self.read[b].record(self.down)
        self.k += 1

    def finish(self):
        """Make the compute stream wait for the last read-backs."""
        for b in range(2):
            self.compute.wait_event(self.read[b])


def main():
    args = parse()
    if args.op == "prefill":
        run_prefill(args)
        return
    if args.op in ("copy_blocks", "swap"):
        run_copy(args)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch(args))
    sp = wl.spec(args.config)
    st = wl.structure(sp)
    world, rank, local = world_of(args)
    if args.impl == "reference":
        run_reference(args, sp, st)
        return

    import torch
    import torch.distributed as dist
    import paged_kv_cache_448_b200 as pk

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    part = sp.partition_tokens if args.partition < 0 else args.partition
    sp_r = dataclasses.replace(sp, seed=rank_seed(sp, rank))
    d = wl.device_data(sp_r, st, device=dev)
    slots = pk.build_slot_mapping(st.block_tables, st.positions, sp.block_size)
    bt = torch.from_numpy(st.block_tables).to(dev)
    cl = torch.from_numpy(sp.context_lens).to(dev)
    sl = torch.from_numpy(slots).to(dev)
    out = torch.empty_like(d["query"])
    max_ctx = int(sp.context_lens.max())
    cdt = pk.dtype_code(d["key_cache"])
    ws = pk.decode_workspace(sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                             sp.block_size, max_ctx, part, device=dev, cache_dtype=cdt)
    eff_part = pk.decode_partition_tokens(sp.num_seqs, sp.num_heads, sp.num_kv_heads,
                                          sp.head_dim, sp.block_size, max_ctx, part, cdt)
    split = eff_part < max_ctx
    launches_per_step = 2 + (1 if split else 0)

    def step(q, nk, nv, btab, ctx, slot, o, ev=None):
        pk.reshape_and_cache(nk, nv, d["key_cache"], d["value_cache"], slot,
                             k_scale=d["k_scale"], v_scale=d["v_scale"])
        if ev is not None:
            ev[0].record()
        pk.decode(o, q, d["key_cache"], d["value_cache"], btab, ctx, max_ctx, sp.scale,
                  k_scale=d["k_scale"], v_scale=d["v_scale"], partition_tokens=part,
                  workspace=ws)
        if ev is not None:
            ev[1].record()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step(d["query"], d["new_key"], d["new_value"], bt, cl, sl, out)
    torch.cuda.synchronize()
    pk.decode_check(ws)

    sampler = ClockSampler(local)
    sampler.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t0.record()
    for k in range(args.steps):
        step(d["query"], d["new_key"], d["new_value"], bt, cl, sl, out, evs[k])
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    elapsed_ms = t0.elapsed_time(t1)
    dec_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    pk.decode_check(ws)

    # e2e: the same step through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        host = {k: d[k].cpu() for k in ("query", "new_key", "new_value")}
        host["bt"] = torch.from_numpy(st.block_tables)
        host["cl"] = torch.from_numpy(sp.context_lens)
        host["sl"] = torch.from_numpy(slots)
        e2e_step = E2EStep(host, out, step, dev)
        e2e_steps = max(1, min(args.steps, 2000))
        for _ in range(3):
            e2e_step()
        e2e_step.finish()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(e2e_steps):
            e2e_step()
        e2e_step.finish()
        b.record()
        torch.cuda.synchronize()
        barrier()
        e2e = {"ms_per_step": a.elapsed_time(b) / e2e_steps, "h2d": e2e_step.h2d,
               "d2h": e2e_step.d2h}
        pk.decode_check(ws)
        # both read-back buffers hold a step's output: the same inputs through
        # the same kernels give the device-timed loop's output, bit for bit
        ref = out.cpu().view(torch.int16)
        for hb in e2e_step.pin_out:
            if not torch.equal(hb.view(torch.int16), ref):
                raise SystemExit("bench.py: an e2e read-back differs from the device-timed output")

    # max over ranks
    step_ms, dec_ms, e2e_ms = max_over_ranks(
        [elapsed_ms / args.steps, dec_ms, e2e["ms_per_step"] if e2e else 0.0], world, dev)
    if e2e:
        e2e["ms_per_step"] = e2e_ms

    if rank == 0:
        line = decode_line(args, sp, st, world, step_ms, dec_ms, eff_part, launches_per_step,
                           clocks, e2e)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(sp, args.cpu_seconds)
        if world == 1 and args.config == 2 and args.partition < 0 and not args.no_rows:
            line["rows"] = run_rows()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
