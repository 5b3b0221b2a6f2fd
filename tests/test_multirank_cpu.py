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


def test_recorded_traffic_is_tied_to_the_decode_sources():
    """roofline.traffic comes from profiles/traffic.json only for the workload
    it was captured on and while the decode kernels' sources (decode_*.cu,
    their headers, api.cu) still hash to the recorded digest."""
    import json

    import bench
    names = {os.path.basename(f) for f in bench.decode_sources()}
    assert {"decode_kernel.cuh", "api.cu", "decode_f16_f16.cu", "decode_reduce.cu"} <= names
    assert "prefill_tc.cu" not in names and "copy_blocks.cu" not in names
    assert bench.recorded_traffic("gqa70b_long") is None
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)["decode"]
    got = bench.recorded_traffic(rec["workload"])
    if rec["sources_sha256"] == bench.sources_digest():
        assert got == rec["dram_read_bytes"] + rec["dram_write_bytes"]
    else:
        assert got is None
