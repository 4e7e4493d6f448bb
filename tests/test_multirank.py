"""bench.py's multi-rank host logic on CPU: two gloo ranks on 127.0.0.1.

The path shards by sequence (every (batch row, kv head) is independent), so
ranks share no data; what crosses ranks is timing and byte totals.  The
checks: the reported time is the slowest rank's, the job's bytes are summed,
every rank draws different inputs, and under the reference arm only rank 0
runs and prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        local_ms = 10.0 * (rank + 1)                 # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, "cpu", world)
        job = bench.sum_over_ranks(1000 * (rank + 1), "cpu", world)
        seed = bench.rank_seed(1234, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        q.put((rank, ms, job, seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_sum_bytes_distinct_seeds():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, job, seeds in got:
        assert ms == 20.0            # max over ranks, seen by every rank
        assert job == 3000.0         # whole-job bytes
        assert len(set(seeds)) == world


def test_single_rank_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu", 1) == 3.5
    assert bench.sum_over_ranks(7, "cpu", 1) == 7.0


@pytest.mark.parametrize("rank", [1])
def test_reference_arm_runs_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_line_on_rank0():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "0", "--steps", "1", "--warmup", "0"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
