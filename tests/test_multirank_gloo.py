"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank of `bench.py --gpus N` runs its own sequence (replicas, weak
scaling); the only cross-rank steps are barriers and the max-over-ranks
reduction of the timed region.  These tests run that logic with the gloo
backend in two spawned processes, plus the reference arm's rank rule."""
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
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from fixed_pattern_sparse_sa_b200 import inputs
        env = {"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)}
        got_env = bench.rank_env(env)
        # per-rank "step times": rank r took 10 + 5 r ms per step over 4 steps
        local_ms = 4 * (10.0 + 5.0 * rank)
        dist.barrier()
        tmax = bench.max_over_ranks(local_ms, "cpu", torch, dist)
        value = bench.aggregate([tmax], [1.0e12 * 4] * world)[0] / 1e12
        # each rank draws its own sequence (seed = rank)
        g = inputs.gen_dsa(1, 64, 2, 1, 64, 2, 32, seed=rank)
        digest = int(g["q_idx"].to(torch.int64).sum().item())
        dist.barrier()
        q.put((rank, got_env, tmax, value, digest))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_max_time_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    slowest = 4 * (10.0 + 5.0 * (world - 1))
    for rank, env, tmax, value, _ in res:
        assert env == (world, rank, rank)
        assert tmax == slowest                      # every rank sees the slowest rank's time
        # whole-job throughput: both ranks' work over the slowest time
        assert value == pytest.approx(world * 4.0 / (slowest / 1e3))
    assert res[0][4] != res[1][4]                   # different sequences per rank


def test_max_over_ranks_without_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.5, "cpu", torch, dist) == 3.5


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_shape():
    """Rank 0's reference line on a tiny row sample carries the contract keys."""
    import argparse
    args = argparse.Namespace(steps=1, warmup=3, cpu_sample_rows=2)
    line = bench.reference_arm(args, 2)
    json.dumps(line)
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    for k in ("metric", "value", "unit", "steps", "warmup", "ms_per_step", "higher_is_better",
              "config", "cpu_baseline", "e2e"):
        assert k in line
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"
