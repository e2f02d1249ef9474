"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, no GPU.

Each rank of `bench.py --gpus N` runs its own decode batch (data-parallel
replicas, weak scaling); the job's time is the slowest rank's and its
throughput counts every rank's bytes.  These tests run that aggregation with
world size 2 over gloo."""
from __future__ import annotations

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # rank r took (r + 1) * 10 ms for its batch; the job took 20 ms
        job_ms = bench.max_over_ranks((rank + 1) * 10.0, world)
        gbs = bench.job_throughput(1_000_000_000, world, job_ms * 1e-3)
        dist.barrier()
        q.put((rank, job_ms, gbs))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_count_all_bytes():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]
    # 2 ranks x 1 GB in 20 ms
    assert res[0][2] == pytest.approx(100.0) and res[1][2] == pytest.approx(100.0)


def test_single_rank_is_the_identity():
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_throughput(2_000_000_000, 1, 0.5) == pytest.approx(4.0)


def _host_case(batch, fp8=False):
    from types import SimpleNamespace
    s = batch.shape
    return SimpleNamespace(batch=batch, fp8=fp8, prologue=s.prologue, Hkv=s.num_kv_heads,
                           D=s.head_dim, k_scale=None, v_scale=None)


def test_oracle_legs_are_time_bounded():
    """The CPU legs of the benchmark: the baseline repeats its sample until a
    time floor is met (plain and prologue workloads); the reference arm sizes
    each step to a run budget."""
    import bench
    from mixed_length_paged_b200 import workloads as W
    leg = bench._cpu_leg(_host_case(W.build("tiny")), [0, 1], 0.05, "tiny")
    assert leg["value"] > 0 and leg["seconds"] >= 0.05 and leg["cores"] >= 1
    pro = W.make_batch(W.DecodeShape("p", 8, 2, 64, prologue=True), [10, 300, 64], seed=3)
    leg = bench._cpu_leg(_host_case(pro), [0, 2], 0.05, "prologue sample")
    assert leg["value"] > 0 and leg["kind"] == "oracle"
    host = bench._host_sample(W.build("tiny"), [0, 1])
    g, dt, toks = bench._cpu_baseline_sample(host, [0, 1])
    assert g > 0 and toks == 237
    # one sequence per step when steps are many, all of them when few
    assert bench._reference_rows(10.0, 2000, 31) == 1
    assert bench._reference_rows(0.5, 4, 31) == 31
    n = bench._reference_rows(0.01, 2001, 31)
    assert n == 7 and n * 0.01 * 2001 <= bench.REF_BUDGET_SECONDS


def test_percentile_and_config_samples():
    import bench
    assert bench._pct(list(range(1, 51)), 0.9) == 45
    assert bench._pct([3.0], 0.9) == 3.0
    assert bench._cpu_rows("fp8", 256)[0] == list(range(0, 256, 4))
    assert bench._cpu_rows("uniform", 64)[0] == list(range(64))
    assert bench.ClockSampler.summarize([None])["sm_mhz"] is None


def test_ab_spread_summary():
    import bench
    t = bench.ABTotals({"x": 0.0})
    t.blocks = {"x": [5.0, 1.0, 4.0, 2.0, 3.0]}
    sp = t.spread("x")
    assert sp == {"block_median_us": 3.0, "block_p90_us": 5.0, "block_min_us": 1.0,
                  "block_max_us": 5.0}
