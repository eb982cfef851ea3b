"""GPU parity: NSA three-branch forward and the IndexCache decode driver."""
import numpy as np
import pytest
import torch

import oracle
from fixed_pattern_sparse_sa_b200 import api, inputs
from _parity import assert_lse_close, assert_out_close, sample_rows, to_dev

pytestmark = pytest.mark.gpu

NSA_CFG = dict(cmp_len=32, cmp_stride=16, sel_block=64, sel_topk=16, window=512)


def _nsa_check(g, out, lse3, sel, rows, cfg):
    """Selection parity with the near-tie rule, then the outputs against the
    oracle's own run: every output and branch LSE on the rows whose block
    choice equals the oracle's; on a near-tie row (its choice differs by
    blocks of equal importance up to 1e-5 of the row maximum) the LSEs of the
    compressed and window branches, which do not depend on the choice."""
    ref = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], rows=rows, **cfg)
    gsel = sel.cpu().numpy().reshape(-1, sel.shape[2], sel.shape[3])[rows]
    same = np.ones(len(rows), dtype=bool)
    for i in range(len(rows)):
        for gg in range(gsel.shape[1]):
            a = set(x for x in gsel[i, gg] if x >= 0)
            b = set(x for x in ref["sel_idx"][i, gg] if x >= 0)
            if a == b:
                continue
            same[i] = False
            imp = ref["imp"][i, gg]
            kth = np.sort(imp[[x for x in b]])[0]           # smallest chosen importance
            tol = 1e-5 * imp.max()
            for blk in a ^ b:
                assert abs(imp[blk] - kth) <= tol, f"row {rows[i]} group {gg}: block {blk} not a near-tie"
    n_diff = int((~same).sum())
    assert n_diff <= max(2, len(rows) // 100), f"{n_diff} near-tie rows"
    B, T, Hq, d = g["q"].shape
    o = out.reshape(-1, Hq, d)[rows]
    l3 = lse3.reshape(-1, Hq, 3)[rows]
    keep = np.nonzero(same)[0]
    assert_out_close(o[keep], ref["out"][keep], "nsa out")
    assert_lse_close(l3[keep], ref["lse_branch"][keep], "nsa lse")
    if n_diff:
        tie = np.nonzero(~same)[0]
        assert_lse_close(l3[tie][..., [0, 2]], ref["lse_branch"][tie][..., [0, 2]], "nsa lse (near ties)")
    return n_diff


@pytest.mark.parametrize("T", [40, 300, 1100])
def test_nsa_small_full_parity(cuda_ok, T):
    g = inputs.gen_nsa(1, T, 32, 2, 64, seed=T)
    gd = to_dev(g)
    out, lse3, sel = api.nsa_fwd(gd["q"], gd["k"], gd["v"], gd["gates"], **NSA_CFG)
    _nsa_check(g, out, lse3, sel, np.arange(T), NSA_CFG)


@pytest.mark.parametrize("T,Hq,Hkv", [(40, 16, 1), (333, 32, 2), (1100, 16, 2), (2000, 48, 4)])
def test_nsa_d128_full_parity(cuda_ok, T, Hq, Hkv):
    # head dim 128 (the tensor-core compressed branch): groups of 16 and 8
    # heads, ragged query blocks, short sequences with no visible block
    g = inputs.gen_nsa(1, T, Hq, Hkv, 128, seed=T + Hq)
    gd = to_dev(g)
    out, lse3, sel = api.nsa_fwd(gd["q"], gd["k"], gd["v"], gd["gates"], **NSA_CFG)
    api.check_device_status()
    _nsa_check(g, out, lse3, sel, np.arange(T), NSA_CFG)


def test_nsa_d128_two_sequences_wide_blocks(cuda_ok):
    # two sequences in one call (batch offsets of Q, the compressed keys and
    # the selection output) and 128-token selection blocks (8 compressed
    # tokens per block instead of 4), window 256
    cfg = dict(cmp_len=32, cmp_stride=16, sel_block=128, sel_topk=4, window=256)
    g = inputs.gen_nsa(2, 1200, 32, 2, 128, seed=11)
    gd = to_dev(g)
    out, lse3, sel = api.nsa_fwd(gd["q"], gd["k"], gd["v"], gd["gates"], **cfg)
    api.check_device_status()
    _nsa_check(g, out, lse3, sel, np.arange(2 * 1200), cfg)


def test_nsa_branches_isolated_by_gates(cuda_ok):
    T = 700
    g = inputs.gen_nsa(1, T, 16, 1, 128, seed=3)
    gd = to_dev(g)
    ref = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], **NSA_CFG)
    for br in range(3):
        oh = torch.zeros_like(gd["gates"])
        oh[..., br] = 1.0
        out, _, sel = api.nsa_fwd(gd["q"], gd["k"], gd["v"], oh, **NSA_CFG)
        # the branch outputs do not depend on the gates; the selected branch
        # is compared on the rows whose block choice equals the oracle's
        same = np.all(np.sort(sel.cpu().numpy().reshape(T, -1), axis=1)
                      == np.sort(ref["sel_idx"].reshape(T, -1), axis=1), axis=1)
        rows = np.arange(T) if br != 1 else np.nonzero(same)[0]
        assert len(rows) >= T - max(2, T // 100)
        assert_out_close(out[0][rows], ref["o_branch"][br][rows], f"branch {br}")
    assert ref["out"].shape == (T, 16, 128)


def test_nsa64k_sampled_rows(cuda_ok):
    w = inputs.WORKLOADS["nsa64k"]
    g = inputs.gen_nsa(w.B, w.T, w.Hq, w.Hkv, w.d, seed=0)
    gd = to_dev(g)
    cfg = dict(cmp_len=w.cmp_len, cmp_stride=w.cmp_stride, sel_block=w.sel_block,
               sel_topk=w.sel_topk, window=w.window)
    out, lse3, sel = api.nsa_fwd(gd["q"], gd["k"], gd["v"], gd["gates"], **cfg)
    rows = sample_rows(w.T, 48, seed=4, edge=8)
    _nsa_check(g, out, lse3, sel, rows, cfg)
    api.check_device_status()


def _decode_layers(nseq, L, n_layers, seed, device="cpu"):
    return [inputs.gen_decode_layer(nseq, L, 16, 1, 128, 8, 64, layer=i, seed=seed, device=device)
            for i in range(n_layers)]


@pytest.mark.parametrize("pattern", ["FSSS", "FFFF", "FSFS"])
def test_indexcache_decode_small(cuda_ok, pattern):
    nseq, L = 3, 5000
    lays = _decode_layers(nseq, L, 4, seed=20)
    dl = [to_dev(x) for x in lays]
    outs, lses, cache = api.dsa_decode_layers(pattern, dl, topk=2048, n_split=8)
    ref = oracle.dsa_layers(pattern, lays, topk=2048)
    for i in range(4):
        assert_out_close(outs[i], ref[i][1], f"layer {i}")
        assert_lse_close(lses[i], ref[i][2], f"layer {i}")
    np.testing.assert_array_equal(cache.cpu().numpy().reshape(ref[-1][0].shape), ref[-1][0])


@pytest.mark.parametrize("n_split", [4, 16])
def test_decode128k_full_size(cuda_ok, n_split):
    # 32 sequences x 131072 cached tokens, 4 layers; caches drawn on the GPU.
    # 4 pieces per row is the benchmark's launch form (CTA-merged pieces).
    w = inputs.WORKLOADS["dsa_decode128k"]
    lays = _decode_layers(w.B, w.T, 4, seed=0, device="cuda")
    for pattern in ("FSSS", "FFFF"):
        outs, lses, cache = api.dsa_decode_layers(pattern, lays, topk=w.topk, n_split=n_split)
        torch.cuda.synchronize()
        # oracle on a few sequences of every layer (host copies of those rows)
        seqs = [0, 17, 31]
        sub = [{k: v[seqs].cpu() for k, v in lay.items()} for lay in lays]
        ref = oracle.dsa_layers(pattern, sub, topk=w.topk)
        for i in range(4):
            assert_out_close(outs[i][seqs], ref[i][1], f"{pattern} layer {i}")
            assert_lse_close(lses[i][seqs], ref[i][2], f"{pattern} layer {i}")
        np.testing.assert_array_equal(cache[seqs].cpu().numpy().reshape(ref[-1][0].shape),
                                      ref[-1][0])
    api.check_device_status()


def _prefill_layers(T, n_layers, seed):
    return [inputs.gen_dsa(1, T, 16, 1, 128, 8, 64, seed=seed + 1000 * i) for i in range(n_layers)]


@pytest.mark.parametrize("pattern", ["FSSS", "FSFS"])
def test_indexcache_prefill_full_parity(cuda_ok, pattern):
    # IndexCache on a prefill (IndexCache page, body: the prefill speed-up
    # comes from S layers skipping the indexer): every query of a 4096-token
    # sequence, 4 layers with independent inputs, top-512.  Indices are
    # bit-exact; every layer's output and LSE match the oracle's layer loop.
    T, topk = 4096, 512
    lays = _prefill_layers(T, 4, seed=30)
    dl = [to_dev(x) for x in lays]
    outs, lses, cache = api.dsa_decode_layers(pattern, dl, topk=topk)
    api.check_device_status()
    ref = oracle.dsa_layers(pattern, lays, topk=topk)
    for i in range(4):
        assert_out_close(outs[i], ref[i][1], f"{pattern} layer {i}")
        assert_lse_close(lses[i], ref[i][2], f"{pattern} layer {i}")
    np.testing.assert_array_equal(cache.cpu().numpy().reshape(ref[-1][0].shape), ref[-1][0])


def test_hysparse2_window128_top1024(cuda_ok):
    # HySparse2 page ("Xiaomi presenta HySparse2 ...", sections "Mas precision
    # con menos memoria" and "Que significa ..."): the 128 most recent tokens
    # are always kept and up to 1024 score-chosen tokens are added.  Every row
    # of an 8192-token prefill: indices bit-exact, attention within tolerance.
    T, topk, window = 8192, 1024, 128
    g = inputs.gen_dsa(1, T, 16, 1, 128, 8, 64, seed=44)
    gd = to_dev(g)
    idx, cnt = api.indexer_topk(gd["q_idx"], gd["k_idx"], gd["w"], topk, window)
    out, lse = api.sparse_attn_fwd(gd["q"], gd["k"], gd["v"], idx)
    api.check_device_status()
    ref_idx, ref_cnt = oracle.indexer_topk(g["q_idx"], g["k_idx"], g["w"], topk, window)
    np.testing.assert_array_equal(cnt.cpu().numpy().reshape(-1), ref_cnt)
    np.testing.assert_array_equal(idx.cpu().numpy().reshape(ref_idx.shape), ref_idx)
    np.testing.assert_array_equal(ref_cnt, np.minimum(np.arange(T) + 1, topk + window))
    rows = sample_rows(T, 512, seed=3)
    ro, rl = oracle.sparse_attn(g["q"], g["k"], g["v"], ref_idx.reshape(1, T, -1), rows=rows)
    assert_out_close(out.reshape(-1, 16, 128)[rows], ro)
    assert_lse_close(lse.reshape(-1, 16)[rows], rl)
