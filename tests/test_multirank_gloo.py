"""Multi-rank host logic on CPU: two gloo ranks.

Each rank of `bench.py --gpus N` runs its own sequence (replicas, weak
scaling); the only cross-rank steps are barriers and the max-over-ranks
reduction of the timed region.  These tests run that logic with the gloo
backend in two spawned processes, plus the reference arm's rank rule.

The sequence-split decode driver (fixed_pattern_sparse_sa_b200.seqsplit)
is run on two gloo ranks as well, with the library calls replaced by
oracle-backed stand-ins: its exchanges and its decomposition (local
top-(k + window) candidates, global merge, partial attention, log-sum-exp
merge) must reproduce the oracle's selection and attention over the whole
sequence."""
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


def _seqsplit_problem(nseq=2, L=3000, topk=200, window=16):
    from fixed_pattern_sparse_sa_b200 import inputs
    lay = inputs.gen_decode_layer(nseq, L, 4, 1, 64, 2, 32, layer=0, seed=3)
    return lay, topk, window


def _seqsplit_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        import _oracle_ops
        from fixed_pattern_sparse_sa_b200 import seqsplit
        lay, topk, window = _seqsplit_problem()
        L = lay["k"].shape[1]
        bounds = [0, 1700, L]                                 # uneven shards
        lo, hi = bounds[rank], bounds[rank + 1]
        sh = seqsplit.Shard(q=lay["q"], k=lay["k"][:, lo:hi], v=lay["v"][:, lo:hi], q_idx=lay["q_idx"],
                            k_idx=lay["k_idx"][:, lo:hi], w=lay["w"], key_lo=lo)
        out, lse, sel = seqsplit.decode_step(sh, topk, window, L, seqsplit.dist_exchange(), bounds[:-1],
                                             ops=_oracle_ops)
        q.put((rank, out.numpy(), lse.numpy(), sel.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
def test_seqsplit_decode_two_gloo_ranks_matches_whole_sequence():
    import numpy as np
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seqsplit_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=200) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    lay, topk, window = _seqsplit_problem()
    L = lay["k"].shape[1]
    ref_idx, _ = oracle.indexer_topk(lay["q_idx"], lay["k_idx"], lay["w"], topk, window, q_pos0=L - 1)
    ro, rl = oracle.sparse_attn(lay["q"], lay["k"], lay["v"], ref_idx.reshape(2, 1, -1), q_pos0=L - 1)
    for rank, out, lse, sel in res:
        np.testing.assert_array_equal(sel.reshape(ref_idx.shape), ref_idx)
        np.testing.assert_allclose(out.reshape(ro.shape), ro, atol=1e-12)
        np.testing.assert_allclose(lse.reshape(rl.shape), rl, atol=1e-12)
