"""The multi-rank path of bench.py on CPU: two gloo ranks (one process each, as torchrun would
start them) agree on the slowest rank's time, the whole-job value counts every replica, and the
reference arm runs on rank 0 alone."""
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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        local_ms = [12.5, 20.0][rank]                      # rank 1 is the slow one
        got = bench.max_over_ranks(local_ms, dist, "cpu")
        dist.barrier()
        q.put((rank, got, bench.replica_value(world, 1_000_000, got / 10)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_both_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    assert [o[1] for o in out] == [20.0, 20.0]              # every rank gets the slowest time
    # 2 replicas x 1 MB per step at 2.0 ms per step = 1.0 GB/s for the whole job
    assert out[0][2] == pytest.approx(1.0) and out[1][2] == pytest.approx(1.0)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
    assert bench.replica_value(1, 2_000_000, 1.0) == pytest.approx(2.0)


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the oracle arm works on rank 0; any other rank exits 0 without output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
