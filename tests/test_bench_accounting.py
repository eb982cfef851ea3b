"""bench.py's work accounting against the oracle's own index sets (CPU).

`value` divides 4*d*Hq*sum_t |S_t| by the step time; the closed form for
sum_t |S_t| used there must equal the number of keys the exact top-k
actually selects."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import oracle  # noqa: E402
from fixed_pattern_sparse_sa_b200 import inputs  # noqa: E402


@pytest.mark.parametrize("T,topk,window", [(300, 64, 0), (300, 64, 16), (200, 256, 8), (97, 1, 0)])
def test_set_sizes_match_the_oracle_topk(T, topk, window):
    g = inputs.gen_dsa(1, T, 2, 1, 64, 2, 32, seed=T + topk)
    _, cnt = oracle.indexer_topk(g["q_idx"], g["k_idx"], g["w"], topk, window)
    assert int(cnt.sum()) == bench.attn_rows(T, topk, window)
    assert bench.attn_flops(T, topk, window, 2, 64) == 4.0 * 64 * 2 * int(cnt.sum())


def test_prefill_64k_flops_constant():
    # the 64K prefill line: top-2048, no forced window, 16 heads, d = 128
    assert bench.attn_flops(65536, 2048, 0, 16, 128) == pytest.approx(1.0823401472e12, rel=1e-9)
    n = 65536
    closed = 2048 * 2049 // 2 + (n - 2048) * 2048
    assert bench.attn_rows(n, 2048, 0) == closed


def test_nsa_flops_match_brute_force_counts():
    # 4*d per (query head, key) summed over the three branches: compressed
    # tokens visible to t, the last `window` keys, and the keys <= t of the
    # blocks the oracle's top-k picked (shared by the heads of a KV group)
    import dataclasses
    import torch
    w = dataclasses.replace(inputs.WORKLOADS["nsa64k"], T=300, Hq=8, Hkv=2, d=64)
    g = inputs.gen_nsa(1, w.T, w.Hq, w.Hkv, w.d, seed=5)
    ref = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], cmp_len=w.cmp_len, cmp_stride=w.cmp_stride,
                         sel_block=w.sel_block, sel_topk=w.sel_topk, window=w.window)
    sel = ref["sel_idx"]                                       # [T, Hkv, k]
    keys = 0
    for t in range(w.T):
        n_cmp = sum(1 for i in range(w.T) if i * w.cmp_stride + w.cmp_len - 1 <= t)
        n_win = min(t + 1, w.window)
        keys += w.Hq * (n_cmp + n_win)
        for gg in range(w.Hkv):
            for blk in sel[t, gg]:
                if blk >= 0:
                    keys += (w.Hq // w.Hkv) * sum(1 for j in range(blk * w.sel_block, (blk + 1) * w.sel_block)
                                                  if j <= t)
    got = bench.nsa_flops(w, torch.from_numpy(sel.reshape(1, w.T, w.Hkv, -1).copy()), torch)
    assert got == 4.0 * w.d * keys
