"""The multi-GPU path of the benchmark on CPU: two gloo ranks.

Sequences are independent, so N GPUs each decode their own batch (weak
scaling) with no collective on the data path; the ranks only agree on the
time (maximum over ranks) and rank 0 reports the whole job's bytes over that
time. This checks that logic with world size 2 on the CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from paged_kv_cache_448_b200 import workloads as wl
        sp = wl.spec(2)
        times = [1.0 + rank, 5.0 - 2 * rank, 0.25 * (rank + 1)]   # per-rank step, decode, e2e ms
        agg = bench.max_over_ranks(times, world, "cpu")
        out.put((rank, agg, bench.rank_seed(sp, rank)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_use_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict()
    for _ in procs:
        rank, agg, seed = q.get(timeout=120)
        res[rank] = (agg, seed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == [2.0, 5.0, 0.5]
    assert res[0][1] != res[1][1]


def _line_worker(rank, world, port, out):
    """One rank of a decode run on CPU stubs: the real seeds, max-over-ranks
    and line assembly of bench.py, with made-up device times."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import argparse

        import bench
        from paged_kv_cache_448_b200 import workloads as wl
        sp = wl.spec(2)
        st = wl.structure(sp)
        args = argparse.Namespace(steps=10, warmup=3, gpus=world)
        # rank 1 is the slower one
        step_ms, dec_ms, e2e_ms = bench.max_over_ranks(
            [0.20 + 0.05 * rank, 0.18 + 0.04 * rank, 0.25 + 0.01 * rank], world, "cpu")
        e2e = {"ms_per_step": e2e_ms, "h2d": 1, "d2h": 2}
        line = bench.decode_line(args, sp, st, world, step_ms, dec_ms, 1024, 3,
                                 {"sm_mhz": None}, e2e) if rank == 0 else None
        out.put((rank, bench.rank_seed(sp, rank), line))
    finally:
        dist.destroy_process_group()


def test_two_rank_decode_line_counts_both_batches_over_the_slowest_rank():
    import bench
    from paged_kv_cache_448_b200 import workloads as wl
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_line_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        rank, seed, line = q.get(timeout=120)
        res[rank] = (seed, line)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] != res[1][0]                     # each rank its own batch
    line = res[0][1]
    sp = wl.spec(2)
    nbytes = wl.decode_bytes(sp, wl.structure(sp))
    assert line["n_gpus"] == 2 and line["config"]["global_batch"] == 2 * sp.num_seqs
    assert line["config"]["parallelism"] == "dp2" and line["scaling"] == "weak"
    assert line["ms_per_step"] == pytest.approx(0.25)
    assert line["value"] == pytest.approx(2 * nbytes / 0.25e-3 / 1e9, rel=1e-3)
    assert line["roofline"]["launch_ms"] == pytest.approx(0.22)
    assert line["e2e"]["value"] == pytest.approx(2 * nbytes / 0.26e-3 / 1e9, rel=1e-3)
    assert bench.job_throughput_gbs(2, nbytes, 0.25) == pytest.approx(line["value"], rel=1e-3)


def test_gpus_n_starts_n_ranks_itself():
    """`python bench.py --gpus 2` without a launcher starts two ranks through
    torch.distributed.run; here on the reference arm, which needs no GPU:
    exactly one JSON line (rank 0's), with n_gpus 2."""
    import json
    import subprocess
    import sys

    import bench
    cmd = bench.relaunch_command(2, 12345, ["--gpus", "2"])
    i = cmd.index("-m")
    assert cmd[:4] == ["timeout", "-k", "60", "3600"]
    assert cmd[i + 1] == "torch.distributed.run" and "--nproc-per-node=2" in cmd
    assert cmd[-3].endswith("bench.py") and cmd[-2:] == ["--gpus", "2"]
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl",
                        "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
                        "--cpu-seconds", "0.2"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["impl"] == "reference"


def test_rank_count_must_match_gpus():
    import argparse

    import bench
    os.environ["WORLD_SIZE"] = "3"
    try:
        with pytest.raises(SystemExit):
            bench.world_of(argparse.Namespace(gpus=2))
    finally:
        del os.environ["WORLD_SIZE"]


def test_job_throughput_counts_every_rank():
    import bench
    one = bench.job_throughput_gbs(1, 1_000_000_000, 100.0)
    assert one == pytest.approx(10.0)
    assert bench.job_throughput_gbs(4, 1_000_000_000, 100.0) == pytest.approx(4 * one)


def test_cpu_baseline_runs_on_one_core_and_on_all_cores():
    """bench.py's cpu_baseline: the oracle single-threaded and on every host
    core (spawned processes behind a barrier), here on the tiny workload and
    on the shared-prefix one (whose samples become private copies)."""
    import bench
    from paged_kv_cache_448_b200 import workloads as wl
    for cfg in (1, 5):
        cb = bench.cpu_baseline(wl.spec(cfg, small=True), 0.5)
        assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0
        allc = cb["all_cores"]
        assert "unavailable" not in allc, allc
        assert allc["cores"] >= 1 and allc["value"] > 0


def test_recorded_traffic_is_tied_to_the_sources():
    """roofline.traffic comes from profiles/traffic.json only for the bench row
    (decode, multi-token query, block copy) and workload it was captured on,
    and while that row's kernel sources (its units, their headers, api.cu)
    still hash to the recorded digest."""
    import json

    import bench
    names = {os.path.basename(f) for f in bench.op_sources("decode")}
    assert {"decode_kernel.cuh", "api.cu", "decode_f16_f16.cu", "decode_reduce.cu",
            "decode_fp8_tc.cu"} <= names
    assert "prefill_tc.cu" not in names and "copy_blocks.cu" not in names
    names = {os.path.basename(f) for f in bench.op_sources("prefill")}
    assert {"prefill_tc.cu", "prefill_kernel.cu", "api.cu", "tc_common.cuh"} <= names
    assert "decode_f16_f16.cu" not in names
    assert {"copy_blocks.cu", "api.cu"} <= {os.path.basename(f)
                                            for f in bench.op_sources("copy_blocks")}
    assert bench.recorded_traffic("no such workload") is None
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)["entries"]
    for e in entries:
        assert e["dram_bytes_per_launch"] == e["dram_read_bytes"] + e["dram_write_bytes"]
        got = bench.recorded_traffic(e["workload"], e["op"])
        if e["sources_sha256"] == bench.sources_digest(e["op"]):
            assert got == e["dram_bytes_per_launch"]
        else:
            assert got is None


def test_rows_run_in_children_and_their_failures_stay_there():
    """bench.py's other rows: each is measured in a child process; its last
    JSON line is summarised, and a child that fails, prints no line or runs
    out of time is reported as such instead of raising, so that the headline
    line is printed whatever a row does. A spent time budget skips the rest."""
    import json
    import sys

    import bench
    line = {"metric": "m", "value": 1.5, "unit": "GB/s", "ms_per_step": 0.1, "dtype": "bf16",
            "roofline": {"bound": "hbm", "achieved": 2.0, "peak": 4.0, "unit": "GB/s",
                         "frac": 0.5, "traffic": None, "peak_kind": "measured", "kernel": "k"},
            "clocks": {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3},
            "config": {"workload": "w"}}
    scripts = {
        "ok": "print('log line'); print(" + repr(json.dumps(line)) + ")",
        "fail": "import sys; print('boom', file=sys.stderr); sys.exit(3)",
        "silent": "pass",
        "slow": "import time; time.sleep(30)",
    }
    rows = [(k, [k]) for k in scripts]

    def command(extra):
        return [sys.executable, "-c", scripts[extra[0]]]

    out = bench.run_rows(rows, budget_s=60, child_timeout_s=3, command=command)
    assert out[0] == {"row": "ok", "metric": "m", "value": 1.5, "unit": "GB/s",
                      "ms_per_step": 0.1, "dtype": "bf16",
                      "roofline": {"bound": "hbm", "achieved": 2.0, "peak": 4.0, "unit": "GB/s",
                                   "frac": 0.5, "traffic": None, "peak_kind": "measured"},
                      "clocks": {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": []}}
    assert out[1]["row"] == "fail" and out[1]["error"] == "exit 3: boom"
    assert out[2]["row"] == "silent" and out[2]["error"].startswith("exit 0")
    assert out[3] == {"row": "slow", "error": "timed out"}
    skipped = bench.run_rows(rows[:2], budget_s=5, child_timeout_s=3, command=command)
    assert [r.get("skipped") for r in skipped] == ["the time budget of the rows was spent"] * 2
    assert [r[0] for r in bench.ROWS][:3] == ["llama13b_mix", "gqa70b_long", "prefix_fp8"]
