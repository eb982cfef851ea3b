"""GPU parity: gathered-KV sparse attention, split-KV partials, LSE combine,
fixed pattern with coordinate bias, device error word."""
import math

import numpy as np
import pytest
import torch

import oracle
from fixed_pattern_sparse_sa_b200 import api, inputs
from fixed_pattern_sparse_sa_b200._lib import SAError
from _parity import assert_lse_close, assert_out_close, sample_rows, to_dev

pytestmark = pytest.mark.gpu


def _random_lists(B, T, heads, K, seed, L=None, q_pos0=0, fill=0.8):
    """Random unsorted index lists inside the causal range, -1 padded."""
    rng = np.random.default_rng(seed)
    L = T if L is None else L
    idx = np.full((B, T, heads, K), -1, dtype=np.int32)
    for b in range(B):
        for t in range(T):
            p = q_pos0 + t
            for h in range(heads):
                n = min(p + 1, int(K * fill) if K > 1 else 1)
                idx[b, t, h, :n] = rng.choice(p + 1, size=n, replace=False)
                rng.shuffle(idx[b, t, h])
    return torch.from_numpy(idx)


def test_tiny_dsa_end_to_end(cuda_ok):
    w = inputs.WORKLOADS["tiny_dsa"]
    g = inputs.gen_dsa(w.B, w.T, w.Hq, w.Hkv, w.d, w.Hi, w.di, seed=0)
    gd = to_dev(g)
    idx, _ = api.indexer_topk(gd["q_idx"], gd["k_idx"], gd["w"], w.topk, w.window)
    out, lse = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], idx)
    ref_idx, _ = oracle.indexer_topk(g["q_idx"], g["k_idx"], g["w"], w.topk, w.window)
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], ref_idx.reshape(1, w.T, -1))
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    api.check_device_status()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(16, 1), (4, 1), (8, 8), (8, 2), (32, 1)])
def test_random_lists(cuda_ok, d, Hq, Hkv):
    B, T, K = 2, 77, 70
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=Hq * 7 + d)
    idx = _random_lists(B, T, 1, K, seed=d + Hq)
    out, lse = api.sparse_attn_fwd(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(), idx.cuda())
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_per_kv_head_lists_and_empty_rows(cuda_ok):
    B, T, Hq, Hkv, d, K = 1, 50, 8, 2, 64, 33
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=3)
    idx = _random_lists(B, T, Hkv, K, seed=4, fill=0.5)
    idx[0, 10:13] = -1                    # empty sets -> zero output, lse = -inf
    out, lse = api.sparse_attn_fwd(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(), idx.cuda())
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    assert torch.all(out[0, 10:13] == 0)


def test_queries_at_the_end_of_a_longer_cache(cuda_ok):
    B, Tq, L, Hq, d, K = 3, 5, 900, 16, 128, 300
    g = inputs.gen_dsa(B, Tq, Hq, 1, d, 1, 32, seed=8, L=L)
    idx = _random_lists(B, Tq, 1, K, seed=9, L=L, q_pos0=L - Tq, fill=1.0)
    out, lse = api.sparse_attn_fwd(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(), idx.cuda())
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, q_pos0=L - Tq)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("n_split", [2, 4, 7, 16])
def test_split_kv_partials_and_combine(cuda_ok, n_split):
    B, Tq, L, Hq, d, K = 4, 1, 3000, 16, 128, 2048
    g = inputs.gen_dsa(B, Tq, Hq, 1, d, 1, 32, seed=10, L=L)
    idx = _random_lists(B, Tq, 1, K, seed=11, L=L, q_pos0=L - 1, fill=1.0)
    out, lse, po, pl = api.sparse_attn_fwd(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(),
                                           idx.cuda(), n_split=n_split, return_partials=True)
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, q_pos0=L - 1)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    # every piece against the oracle on that piece alone
    c = -(-K // n_split)
    for s in range(n_split):
        part = torch.full_like(idx, -1)
        part[..., s * c:(s + 1) * c] = idx[..., s * c:(s + 1) * c]
        so, sl = oracle.sparse_attn(g["q"], g["k"], g["v"], part, q_pos0=L - 1)
        np.testing.assert_allclose(po[s].cpu().numpy().reshape(so.shape), so, atol=2e-3)
        assert_lse_close(pl[s], sl)
    # the standalone combine call on the same partials
    o2, l2 = api.lse_combine(po, pl)
    assert_out_close(o2, ro)
    assert_lse_close(l2, rl)


@pytest.mark.parametrize("Hq,Hkv,idx_heads", [(16, 1, 1), (8, 2, 2), (12, 1, 1)])
def test_d128_empty_rows_ragged_lists_and_bad_index(cuda_ok, Hq, Hkv, idx_heads):
    # head dim 128 with at most 16 heads per KV head (the tensor-core gather
    # path): several 128-key tiles plus a ragged tail, empty rows, a future
    # index that must be reported and skipped
    B, T, d, K = 2, 300, 128, 290
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=21 + Hq)
    idx = _random_lists(B, T, idx_heads, K, seed=22 + Hq, fill=0.9)
    idx[1, 40:43] = -1
    out, lse = api.sparse_attn_fwd(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(), idx.cuda())
    api.check_device_status()
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    assert torch.all(out[1, 40:43] == 0)
    bad = idx.clone()
    bad[0, 5, 0, 0] = 7                    # query 5 cannot see position 7
    out2, _ = api.sparse_attn_fwd(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(), bad.cuda())
    with pytest.raises(SAError):
        api.check_device_status()
    skip = bad.clone(); skip[0, 5, 0, 0] = -1
    ro2, _ = oracle.sparse_attn(g["q"], g["k"], g["v"], skip)
    assert_out_close(out2, ro2)


@pytest.mark.parametrize("n_split", [1, 3])
def test_tensor_core_gather_path(cuda_ok, n_split):
    # the opt-in tcgen05 gather kernel (SA_ATTN_PATH=tc), in a fresh process:
    # ragged lists, empty rows, G = 12 and 16, split pieces
    import subprocess, sys, os
    code = (
        "import torch, numpy as np, oracle\n"
        "from fixed_pattern_sparse_sa_b200 import api, inputs\n"
        "import sys; sys.path.insert(0, 'tests')\n"
        "from _parity import assert_out_close, assert_lse_close\n"
        "from test_gpu_attn import _random_lists\n"
        "for Hq, seed in ((16, 41), (12, 42)):\n"
        "    g = inputs.gen_dsa(2, 300, Hq, 1, 128, 1, 32, seed=seed)\n"
        "    idx = _random_lists(2, 300, 1, 290, seed=seed + 1, fill=0.9)\n"
        "    idx[1, 40:43] = -1\n"
        f"    out, lse = api.sparse_attn_fwd(g['q'].cuda(), g['k'].cuda(), g['v'].cuda(), idx.cuda(), n_split={n_split})\n"
        "    api.check_device_status()\n"
        "    ro, rl = oracle.sparse_attn(g['q'], g['k'], g['v'], idx)\n"
        "    assert_out_close(out, ro); assert_lse_close(lse, rl)\n"
        "print('ok')\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SA_ATTN_PATH="tc")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stderr[-2000:]


def test_lse_combine_with_empty_pieces(cuda_ok):
    S, R, d = 5, 37, 64
    rng = np.random.default_rng(12)
    po = rng.standard_normal((S, R, d)).astype(np.float32)
    pl = rng.standard_normal((S, R)).astype(np.float32) * 3
    pl[1] = -np.inf
    pl[:, 3] = -np.inf                    # a row with nothing at all
    out, lse = api.lse_combine(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda())
    ro, rl = oracle.lse_combine(po, pl)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("T,H,Hkv,d", [(700, 2, 2, 64), (300, 16, 1, 128), (1000, 4, 2, 64)])
def test_fixed_pattern_with_bias(cuda_ok, T, H, Hkv, d):
    g = inputs.gen_spatial(1, T, H, d, beta=0.5, seed=T, Hkv=Hkv)
    gd = to_dev(g)
    out, lse = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], pattern=(65, True),
                                   cq=gd["cq"], ck=gd["ck"], beta=gd["beta"])
    idx, _ = oracle.fixed_graph(T, 65, True, cap=100)
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx.reshape(1, T, -1),
                                cq=g["cq"], ck=g["ck"], beta=g["beta"])
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    # pattern without bias, window only
    out2, lse2 = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], pattern=(9, False))
    idx2, _ = oracle.fixed_graph(T, 9, False, cap=9)
    ro2, rl2 = oracle.sparse_attn(g["q"], g["k"], g["v"], idx2.reshape(1, T, -1))
    assert_out_close(out2, ro2)
    assert_lse_close(lse2, rl2)


def test_spatial16k_full_parity(cuda_ok):
    w = inputs.WORKLOADS["spatial16k"]
    g = inputs.gen_spatial(w.B, w.T, w.Hq, w.d, beta=w.beta, seed=0)
    gd = to_dev(g)
    out, lse = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], pattern=(w.window, w.dilated),
                                   cq=gd["cq"], ck=gd["ck"], beta=gd["beta"])
    idx, cnt = oracle.fixed_graph(w.T, w.window, w.dilated, cap=80)
    assert int(cnt.sum()) == 1161305
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx.reshape(1, w.T, -1),
                                cq=g["cq"], ck=g["ck"], beta=g["beta"])
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_prefill64k_attention_sampled_rows(cuda_ok):
    # full-size run in the launch configuration the benchmark times
    w = inputs.WORKLOADS["dsa_prefill64k"]
    g = inputs.gen_dsa(w.B, w.T, w.Hq, w.Hkv, w.d, w.Hi, w.di, seed=0)
    gd = to_dev(g)
    idx, _ = api.indexer_topk(gd["q_idx"], gd["k_idx"], gd["w"], w.topk, w.window)
    out, lse = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], idx)
    rows = sample_rows(w.T, 192, seed=2)
    ref_idx, _ = oracle.indexer_topk(g["q_idx"], g["k_idx"], g["w"], w.topk, w.window, rows=rows)
    np.testing.assert_array_equal(idx[0].cpu().numpy()[rows], ref_idx)
    full = np.full((1, w.T, ref_idx.shape[-1]), -1, dtype=np.int32)     # the oracle's own sets
    full[0, rows] = ref_idx
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], full, rows=rows)
    assert_out_close(out[0][rows], ro)
    assert_lse_close(lse[0][rows], rl)
    assert torch.isfinite(out.float()).all()
    api.check_device_status()


def test_bad_index_sets_device_error_word(cuda_ok):
    B, T, Hq, d = 1, 8, 16, 64
    g = inputs.gen_dsa(B, T, Hq, 1, d, 1, 32, seed=13)
    idx = torch.full((B, T, 4), -1, dtype=torch.int32)
    for t in range(T):
        idx[0, t, 0] = t
    idx[0, 2, 1] = 5                       # a future position for query 2
    out, _ = api.sparse_attn_fwd(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(), idx.cuda())
    with pytest.raises(SAError) as ei:
        api.check_device_status()
    assert ei.value.status == 5
    api.check_device_status()              # the word was cleared
    # the offending entry was skipped: row 2 equals attention over {2} alone
    idx2 = idx.clone(); idx2[0, 2, 1] = -1
    ro, _ = oracle.sparse_attn(g["q"], g["k"], g["v"], idx2)
    assert_out_close(out, ro)


@pytest.mark.parametrize("scale", [-0.3, 0.0, 0.21])
@pytest.mark.parametrize("d,Hq", [(128, 16), (64, 4)])
def test_explicit_scale_signs(cuda_ok, scale, d, Hq):
    """Any scale, including negative (folded into Q's sign) and zero (uniform
    weights over each row's keys); ragged lists leave partial chunks whose
    empty entries must get exactly zero weight."""
    B, T, K = 1, 90, 45
    g = inputs.gen_dsa(B, T, Hq, 1, d, 1, 32, seed=int(scale * 100) + d)
    idx = _random_lists(B, T, 1, K, seed=d + 5, fill=0.7)
    out, lse = api.sparse_attn_fwd(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(), idx.cuda(), scale=scale)
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, scale=scale)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("scale", [-0.15, 0.0])
def test_fixed_pattern_bias_with_explicit_scale(cuda_ok, scale):
    T, H, d = 300, 16, 128
    g = inputs.gen_spatial(1, T, H, d, beta=0.5, seed=11)
    gd = to_dev(g)
    out, lse = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], pattern=(65, True), cq=gd["cq"], ck=gd["ck"],
                                   beta=gd["beta"], scale=scale)
    idx, _ = oracle.fixed_graph(T, 65, True, cap=100)
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx.reshape(1, T, -1), cq=g["cq"], ck=g["ck"],
                                beta=g["beta"], scale=scale)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_sa_log_prints_launch_configs(cuda_ok):
    """SA_LOG=1 prints one line per kernel launch with its grid, block and
    shared memory (checked in a child process so the setting stays local)."""
    import os
    import subprocess
    import sys
    code = ("import torch\n"
            "from fixed_pattern_sparse_sa_b200 import api, inputs\n"
            "g = inputs.gen_dsa(1, 40, 16, 1, 128, 1, 32, seed=1)\n"
            "idx = torch.randint(0, 40, (1, 40, 8), dtype=torch.int32)\n"
            "idx = torch.where(idx <= torch.arange(40).view(1, 40, 1), idx, torch.full_like(idx, -1))\n"
            "api.sparse_attn_fwd(g['q'].cuda(), g['k'].cuda(), g['v'].cuda(), idx.cuda())\n"
            "torch.cuda.synchronize()\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SA_LOG="1", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stderr.splitlines() if ln.startswith("[sa] ")]
    assert any("gather_attn" in ln or "launch_gather" in ln for ln in lines), r.stderr[-2000:]
    assert all("grid=(" in ln and "block=(" in ln and "smem=" in ln for ln in lines)


@pytest.mark.parametrize("window", [17, 40, 65, 100])
def test_fixed_pattern_one_head_per_kv_windows(cuda_ok, window):
    """One query head per KV head, d = 64: windows whose band fills whole
    16-key chunks take the dilated keys on the CUDA cores, the others on
    the tensor cores; both must match the oracle, with and without bias."""
    T, H, d = 900, 4, 64
    g = inputs.gen_spatial(1, T, H, d, beta=0.5, seed=window, Hkv=H)
    gd = to_dev(g)
    idx, _ = oracle.fixed_graph(T, window, True, cap=window + 16)
    out, lse = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], pattern=(window, True), cq=gd["cq"], ck=gd["ck"],
                                   beta=gd["beta"])
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], idx.reshape(1, T, -1), cq=g["cq"], ck=g["ck"],
                                beta=g["beta"])
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    out2, lse2 = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], pattern=(window, True))
    ro2, rl2 = oracle.sparse_attn(g["q"], g["k"], g["v"], idx.reshape(1, T, -1))
    assert_out_close(out2, ro2)
    assert_lse_close(lse2, rl2)
