"""GPU parity: indexer scores + exact causal top-k (bit-exact indices)."""
import numpy as np
import pytest
import torch

import oracle
from fixed_pattern_sparse_sa_b200 import api, inputs
from _parity import sample_rows, to_dev

pytestmark = pytest.mark.gpu


def _check_rows(got_idx, got_cnt, ref_idx, ref_cnt, rows=None):
    gi = got_idx.cpu().numpy().reshape(-1, got_idx.shape[-1])
    gc = got_cnt.cpu().numpy().reshape(-1)
    if rows is not None:
        gi, gc = gi[rows], gc[rows]
    np.testing.assert_array_equal(gc, ref_cnt)
    np.testing.assert_array_equal(gi, ref_idx)


def test_tiny_dsa_topk_bit_exact(cuda_ok):
    w = inputs.WORKLOADS["tiny_dsa"]
    g = inputs.gen_dsa(w.B, w.T, w.Hq, w.Hkv, w.d, w.Hi, w.di, seed=0)
    gd = to_dev(g)
    idx, cnt = api.indexer_topk(gd["q_idx"], gd["k_idx"], gd["w"], w.topk, w.window)
    ref_idx, ref_cnt = oracle.indexer_topk(g["q_idx"], g["k_idx"], g["w"], w.topk, w.window)
    _check_rows(idx, cnt, ref_idx, ref_cnt)
    api.check_device_status()


@pytest.mark.parametrize("T", [1, 2, 17, 63, 64, 65, 127, 128, 129, 300])
@pytest.mark.parametrize("Hi,di", [(2, 32), (8, 64), (1, 128), (4, 32), (16, 64)])
def test_ragged_shapes_bit_exact(cuda_ok, T, Hi, di):
    g = inputs.gen_dsa(2, T, 1, 1, 64, Hi, di, seed=T * 31 + Hi)
    gd = to_dev(g)
    for topk, window in [(16, 0), (5, 4), (T, 0), (40, 8)]:
        idx, cnt = api.indexer_topk(gd["q_idx"], gd["k_idx"], gd["w"], topk, window)
        ref_idx, ref_cnt = oracle.indexer_topk(g["q_idx"], g["k_idx"], g["w"], topk, window)
        _check_rows(idx, cnt, ref_idx, ref_cnt)


def test_heavy_ties_bit_exact(cuda_ok):
    # tiny value range and mostly-zero weights: huge tie groups at the threshold
    gen = torch.Generator().manual_seed(5)
    B, T, Hi, di = 1, 700, 8, 32
    q = torch.randint(-1, 2, (B, T, Hi, di), generator=gen).to(torch.int8)
    k = torch.randint(-1, 2, (B, T, di), generator=gen).to(torch.int8)
    w = (torch.rand((B, T, Hi), generator=gen) < 0.2).to(torch.int32)
    idx, cnt = api.indexer_topk(q.cuda(), k.cuda(), w.cuda(), 64, 16)
    ref_idx, ref_cnt = oracle.indexer_topk(q, k, w, 64, 16)
    _check_rows(idx, cnt, ref_idx, ref_cnt)


def test_wide_value_range_and_negative_weights(cuda_ok):
    # large int8 magnitudes and signed weights: scores span > 2^24, forcing
    # three radix digit passes and negative keys
    gen = torch.Generator().manual_seed(6)
    B, T, Hi, di = 1, 400, 4, 128
    q = torch.randint(-128, 128, (B, T, Hi, di), generator=gen).to(torch.int8)
    k = torch.randint(-128, 128, (B, T, di), generator=gen).to(torch.int8)
    w = torch.randint(-300, 301, (B, T, Hi), generator=gen).to(torch.int32)
    idx, cnt = api.indexer_topk(q.cuda(), k.cuda(), w.cuda(), 50, 0)
    ref_idx, ref_cnt = oracle.indexer_topk(q, k, w, 50, 0)
    _check_rows(idx, cnt, ref_idx, ref_cnt)


def test_decode_rows_multi_cta_clusters(cuda_ok):
    # one query per sequence at the last position: decode-shaped score pass
    # (tensor-core mma.sync) and the 1024-thread select (one CTA per row)
    nseq, L = 4, 40000
    g = inputs.gen_decode_layer(nseq, L, 16, 1, 128, 8, 64, layer=0, seed=7)
    gd = to_dev(g)
    idx, cnt = api.indexer_topk(gd["q_idx"], gd["k_idx"], gd["w"], 2048, 0)
    ref_idx, ref_cnt = oracle.indexer_topk(g["q_idx"], g["k_idx"], g["w"], 2048, 0, q_pos0=L - 1)
    _check_rows(idx, cnt, ref_idx, ref_cnt)


@pytest.mark.parametrize("Hi,di,wlo,whi", [(8, 64, -300, 301), (8, 64, 0, 40), (4, 32, -3, 4), (1, 64, 0, 200)])
def test_prefill_rows_signed_and_wide_weights(cuda_ok, Hi, di, wlo, whi):
    # prefill shapes with weights that cannot be folded into the query (the
    # filter pass then multiplies per head), over several 128-row blocks and
    # a ragged last block, with and without a forced window
    gen = torch.Generator().manual_seed(60 + Hi + whi)
    B, T = 2, 1000
    q = torch.randint(-128, 128, (B, T, Hi, di), generator=gen).to(torch.int8)
    k = torch.randint(-128, 128, (B, T, di), generator=gen).to(torch.int8)
    w = torch.randint(wlo, whi, (B, T, Hi), generator=gen).to(torch.int32)
    for topk, window in [(64, 0), (200, 32)]:
        idx, cnt = api.indexer_topk(q.cuda(), k.cuda(), w.cuda(), topk, window)
        ref_idx, ref_cnt = oracle.indexer_topk(q, k, w, topk, window)
        _check_rows(idx, cnt, ref_idx, ref_cnt)
    api.check_device_status()


@pytest.mark.parametrize("Tq,wlo,whi", [(1, -300, 301), (2, 0, 40), (1, 0, 5)])
def test_decode_shaped_calls_fold_and_signed_weights(cuda_ok, Tq, wlo, whi):
    # 8 indexer heads of width 64 with one or two queries per sequence (the
    # tensor-core decode scorer): weights that fold into the query operand,
    # weights whose product with q leaves int8, and negative weights
    gen = torch.Generator().manual_seed(40 + Tq + whi)
    B, L, Hi, di = 3, 20000, 8, 64
    q = torch.randint(-128, 128, (B, Tq, Hi, di), generator=gen).to(torch.int8)
    k = torch.randint(-128, 128, (B, L, di), generator=gen).to(torch.int8)
    w = torch.randint(wlo, whi, (B, Tq, Hi), generator=gen).to(torch.int32)
    for topk, window in [(2048, 0), (300, 64)]:
        idx, cnt = api.indexer_topk(q.cuda(), k.cuda(), w.cuda(), topk, window, q_pos0=L - Tq)
        ref_idx, ref_cnt = oracle.indexer_topk(q, k, w, topk, window, q_pos0=L - Tq)
        _check_rows(idx, cnt, ref_idx, ref_cnt)
    api.check_device_status()


def test_prefill64k_sampled_rows_bit_exact(cuda_ok):
    w = inputs.WORKLOADS["dsa_prefill64k"]
    g = inputs.gen_dsa(w.B, w.T, w.Hq, w.Hkv, w.d, w.Hi, w.di, seed=0)
    gd = to_dev(g)
    idx, cnt = api.indexer_topk(gd["q_idx"], gd["k_idx"], gd["w"], w.topk, w.window)
    rows = sample_rows(w.T, 192, seed=1)
    ref_idx, ref_cnt = oracle.indexer_topk(g["q_idx"], g["k_idx"], g["w"], w.topk, w.window,
                                           rows=rows)
    _check_rows(idx, cnt, ref_idx, ref_cnt, rows=rows)
    # properties that hold for every row
    c = cnt.cpu().numpy()[0]
    np.testing.assert_array_equal(c, np.minimum(np.arange(w.T) + 1, w.topk))
    ii = idx[0].cpu().numpy()
    valid = ii >= 0
    assert np.all(ii[valid] <= np.repeat(np.arange(w.T)[:, None], ii.shape[1], 1)[valid])
    d = np.diff(np.where(valid, ii, np.iinfo(np.int32).max).astype(np.int64), axis=1)
    assert np.all(d[valid[:, 1:]] > 0), "rows must be strictly ascending"


def _recompute_case(kind, Tq, L, topk, window, Hi=8, di=64):
    """Inputs on which the sampled threshold cannot give a usable candidate
    list.  "overflow": every weight is 0, so every score ties at 0 and every
    candidate reaches the threshold.  "short": scores are high only on every
    18th key, so half of the positions sampled with stride 9 are high, the
    threshold sits at the high score and only ~1/18 of the row (fewer than
    topk keys) reaches it."""
    gen = torch.Generator().manual_seed(90 + Tq + window)
    if kind == "overflow":
        q = torch.randint(-8, 9, (1, Tq, Hi, di), generator=gen).to(torch.int8)
        k = torch.randint(-8, 9, (1, L, di), generator=gen).to(torch.int8)
        w = torch.zeros((1, Tq, Hi), dtype=torch.int32)
    else:
        q = torch.ones((1, Tq, Hi, di), dtype=torch.int8)
        k = torch.ones((1, L, di), dtype=torch.int8)
        k[0, ::18] = 2
        w = torch.ones((1, Tq, Hi), dtype=torch.int32)
    return q, k, w


@pytest.mark.parametrize("kind", ["overflow", "short"])
@pytest.mark.parametrize("Tq", [64, 1])
@pytest.mark.parametrize("window", [0, 64])
def test_exact_recompute_when_sample_fails(cuda_ok, kind, Tq, window):
    # L = 20000 makes the sample strided (stride 9 for these rows): the exact
    # answer must not depend on it.  Tq = 64 runs the tcgen05 score passes,
    # Tq = 1 the decode-shaped ones; both end in the select kernel's exact
    # recompute, which the device counter confirms.
    L, topk = 20000, 2048
    q, k, w = _recompute_case(kind, Tq, L, topk, window)
    api.debug_exact_recompute_rows()                     # clear the counter
    idx, cnt = api.indexer_topk(q.cuda(), k.cuda(), w.cuda(), topk, window, q_pos0=L - Tq)
    n_re = api.debug_exact_recompute_rows()
    ref_idx, ref_cnt = oracle.indexer_topk(q, k, w, topk, window, q_pos0=L - Tq)
    _check_rows(idx, cnt, ref_idx, ref_cnt)
    assert n_re == Tq, f"{n_re} of {Tq} rows took the exact-recompute path"
    api.check_device_status()
