"""World-size-2 checks of bench.py's multi-rank host logic on CPU (gloo).

With N GPUs the bench runs N independent replicas of the prefill layer: each rank times its
own steps, the step time reported is the maximum over ranks, the throughput is summed over
ranks, and only rank 0 prints.  No collective sits on the data path; the ones here only
synchronise and reduce timings, exactly as bench.py does under torchrun with NCCL.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_env()
        assert (w, r, lr) == (world, rank, rank)
        bench.barrier(w)
        # each rank "measured" a different step time; everyone must see the slowest
        mine = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(mine, w, torch.device("cpu"))
        rate = bench.whole_job_rate(w, 2176, mx)
        q.put((rank, mine, mx, rate))
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    slowest = 10.0 + 5.0 * (world - 1)
    for rank, mine, mx, rate in got:
        assert mx == slowest                                  # max over ranks, seen by every rank
        assert rate == pytest.approx(world * 2176 / (slowest * 1e-3))   # summed over replicas


def test_single_rank_helpers_without_process_group():
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.whole_job_rate(1, 1000, 2.0) == pytest.approx(5e5)
    bench.barrier(1)   # no-op


def test_reference_arm_nonzero_rank_exits_without_work():
    """Under torchrun the reference arm runs on rank 0 only; other ranks exit 0, print nothing."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_time_oracle_small_sample():
    """The cpu_baseline leg times the oracle on a bounded sample of the SWA workload."""
    rate, el, reps = bench.time_oracle(16, 0.0)
    assert rate > 0 and reps >= 1 and el > 0


def test_reference_arm_runs_exactly_the_reported_steps():
    """The reference arm times exactly `steps` oracle steps after `warmup` untimed ones, each a
    bounded sample of the workload (here the smallest, 64 input tokens)."""
    rate, ms, n, el = bench.reference_steps(2, 1, total_budget_s=0.0)
    assert n == 64 and rate > 0
    assert ms == pytest.approx(1000.0 * el / 2)
