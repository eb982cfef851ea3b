"""GPU parity of the full-attention layer used as an exact indexer
(sa_full_attn_topk; HySparse2 page, "Que significa para la evolucion de la
IA" and "Mas precision con menos memoria") against the fp64 oracle.

The full layer's output and LSE are compared with the attention tolerance
of the other paths (per element |got - ref| <= 1e-2 + 2^-8 |ref|, LSE
1e-3).  The index sets: the forced window must match exactly; the score
part is compared with the oracle's set row by row, and where a row differs
every key the GPU chose must score, in fp64, at least the oracle's k-th
score less the fp32 error bound, and every key it left out at most that
score plus the bound.  The bound: each logit is an fp32 sum of d bf16
products (relative error <= d * 2^-24 of the sum of magnitudes, ~1e-4 of
the exponent at these sizes) and the LSE comes from the fp32 attention, so
a score moves by at most 2e-4 of itself; at most 2 % of the rows may
differ."""
import math

import numpy as np
import pytest
import torch

import oracle
from fixed_pattern_sparse_sa_b200 import api, inputs

pytestmark = pytest.mark.gpu

REL = 2e-4


def _check_out(out, lse, ref_out, ref_lse, rows=None):
    o = out.float().cpu().numpy().reshape(-1, *out.shape[2:])
    l = lse.cpu().numpy().reshape(-1, lse.shape[-1])
    if rows is not None:
        o, l = o[rows], l[rows]
    assert np.all(np.abs(o - ref_out) <= 1e-2 + 2.0 ** -8 * np.abs(ref_out))
    assert np.abs(l - ref_lse).max() <= 1e-3


def _check_sets(idx, ref_idx, sc, topk, window, T, rows):
    """idx / ref_idx [n, topk+window], sc [n, T] fp64 oracle scores."""
    g = idx.cpu().numpy().reshape(-1, idx.shape[-1])[rows] if rows is not None else \
        idx.cpu().numpy().reshape(-1, idx.shape[-1])
    differ = 0
    for i in range(g.shape[0]):
        t = int(rows[i]) % T if rows is not None else i % T
        if np.array_equal(g[i], ref_idx[i]):
            continue
        differ += 1
        w_lo = max(0, t - window + 1) if window > 0 else t + 1
        got = g[i][g[i] >= 0]
        # window part exact, order ascending, no repeats, causal
        assert np.all(np.diff(got) > 0) and got.max() <= t
        assert np.array_equal(got[got >= w_lo], np.arange(w_lo, t + 1))
        chosen = got[got < w_lo]
        assert len(chosen) == min(topk, w_lo)
        kth = np.sort(sc[i, :w_lo])[::-1][len(chosen) - 1]
        tol = REL * kth + 1e-9
        assert np.all(sc[i, chosen] >= kth - tol)
        rest = np.setdiff1d(np.arange(w_lo), chosen)
        if len(rest):
            assert np.all(sc[i, rest] <= kth + tol)
    assert differ <= max(1, int(0.02 * g.shape[0])), f"{differ} rows differ"


@pytest.mark.parametrize("B,T,Hq,Hkv,d,topk,window", [
    (1, 300, 16, 1, 128, 64, 16),       # MQA, tcgen05 full layer
    (2, 257, 8, 2, 64, 40, 8),          # two KV groups summed, d = 64, ragged chunks
    (1, 200, 12, 1, 128, 300, 20),      # k larger than the candidates: all kept
    (1, 130, 4, 4, 64, 16, 0),          # no window
    (1, 2065, 16, 1, 128, 1024, 128),   # the HySparse2 selection, ragged, several score chunks of keys
    (1, 700, 32, 2, 128, 100, 32),      # two KV groups of 16 heads on the tcgen05 score pass
    (2, 333, 16, 1, 128, 50, 0),        # two sequences, no window, ragged query blocks
    (2, 450, 64, 4, 128, 60, 8),        # four KV groups of 16 heads, two sequences
])
def test_full_attn_indexer_parity(cuda_ok, B, T, Hq, Hkv, d, topk, window):
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=T + d)
    q, k, v = g["q"], g["k"], g["v"]
    out, lse, idx = api.full_attn_topk(q.cuda(), k.cuda(), v.cuda(), topk, window)
    api.check_device_status()
    ref_out, ref_lse, ref_idx, sc = oracle.full_attn_topk(q, k, v, topk, window, want_scores=True)
    _check_out(out, lse, ref_out, ref_lse)
    _check_sets(idx, ref_idx, sc, topk, window, T, None)


def test_full_attn_indexer_16k_sampled_rows(cuda_ok):
    # the shape of the HySparse2 selection (window 128 + top-1024) on a
    # 16384-token prefill, 16 query heads sharing one KV head, d = 128;
    # sampled rows against the oracle, every row's format checked
    B, T, Hq, Hkv, d, topk, window = 1, 16384, 16, 1, 128, 1024, 128
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=11)
    q, k, v = g["q"], g["k"], g["v"]
    out, lse, idx = api.full_attn_topk(q.cuda(), k.cuda(), v.cuda(), topk, window)
    api.check_device_status()
    rows = np.array([0, 1, 127, 128, 1151, 1152, 1153, 5000, 9999, T - 2, T - 1])
    ref_out, ref_lse, ref_idx, sc = oracle.full_attn_topk(q, k, v, topk, window, rows=rows,
                                                          want_scores=True)
    _check_out(out, lse, ref_out, ref_lse, rows)
    _check_sets(idx, ref_idx, sc, topk, window, T, rows)
    ii = idx[0]
    cnt = (ii >= 0).sum(dim=1).cpu()
    t = torch.arange(T)
    assert torch.equal(cnt, torch.clamp(t + 1, max=topk + window))
    valid = ii >= 0
    assert torch.all(valid[:, :-1] | ~valid[:, 1:])             # entries first, then padding
    assert torch.all((ii[:, 1:] > ii[:, :-1]) | ~valid[:, 1:])  # ascending
    assert torch.all(ii.max(dim=1).values.cpu() == t)


def test_full_attn_indexer_32k_row_chunks(cuda_ok):
    # 32768 tokens: the dense scores are taken in four chunks of 8192 query
    # rows (1 GiB each); sampled rows on both sides of every chunk boundary
    B, T, Hq, Hkv, d, topk, window = 1, 32768, 16, 1, 128, 1024, 128
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=12)
    q, k, v = g["q"], g["k"], g["v"]
    out, lse, idx = api.full_attn_topk(q.cuda(), k.cuda(), v.cuda(), topk, window)
    api.check_device_status()
    rows = np.array([3, 8191, 8192, 8193, 16383, 16384, 24575, 24576, T - 1])
    ref_out, ref_lse, ref_idx, sc = oracle.full_attn_topk(q, k, v, topk, window, rows=rows,
                                                          want_scores=True)
    _check_out(out, lse, ref_out, ref_lse, rows)
    _check_sets(idx, ref_idx, sc, topk, window, T, rows)
    cnt = (idx[0] >= 0).sum(dim=1).cpu()
    assert torch.equal(cnt, torch.clamp(torch.arange(T) + 1, max=topk + window))
