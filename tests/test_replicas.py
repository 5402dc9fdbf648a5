"""The multi-GPU plumbing of bench.py on the CPU: N ranks run independent
replicas of the layer, and the process group carries only the barriers and the
max-over-ranks reduction of the timings.  Run here as world_size-2 `gloo` ranks.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, _ = bench.dist_env()
    bench.init_replicas(w, "gloo", timeout_s=30)
    try:
        # rank-dependent timings: step ms, K1, K2, K3, e2e
        mine = [1.0 + r, 0.1 * (w - r), 0.5, 0.25 + 0.01 * r, 3.0 - r]
        dist.barrier()
        got = bench.max_over_ranks(mine, w)
        out.put((r, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [2.0, 0.2, 0.5, 0.26, 3.0]
    for r in (0, 1):
        assert res[r] == pytest.approx(want)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]


def test_aggregate_counts_every_replica_over_the_slowest_step():
    # 2 replicas of 1e12 FLOP each, slowest rank 0.5 ms per step -> 4000 TFLOP/s
    assert bench.aggregate_tflops(1e12, 2, 0.5) == pytest.approx(4000.0)
    assert bench.aggregate_tflops(1e12, 1, 0.5) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
