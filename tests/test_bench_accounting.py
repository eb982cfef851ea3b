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
