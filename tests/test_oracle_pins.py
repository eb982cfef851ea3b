"""Pins for the CPU oracle: each oracle function is checked against something
other than itself -- torch float64 scaled_dot_product_attention, numpy
einsum / lexsort, hand-derived sets, closed forms and invariants -- chosen so
that a dropped term, a wrong sign or index, or a transposed operand fails.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from fixed_pattern_sparse_sa_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers --
def _f64(t):
    return t.to(torch.float64)


def sdpa_ref(q, k, v, mask=None, scale=None):
    """torch float64 SDPA.  q [B,T,Hq,d], k/v [B,L,Hkv,d]; mask broadcastable
    to [B,Hq,T,L] (bool: True = attend, or float additive)."""
    qh = _f64(q).transpose(1, 2)
    kh = _f64(k).transpose(1, 2)
    vh = _f64(v).transpose(1, 2)
    o = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask, scale=scale,
                                       enable_gqa=True)
    return o.transpose(1, 2).numpy()


def lse_ref(q, k, mask_bool, scale, bias=None):
    """logsumexp of the masked logits with torch (float64)."""
    qh = _f64(q).transpose(1, 2)
    kh = _f64(k).transpose(1, 2)
    G = qh.shape[1] // kh.shape[1]
    kh = kh.repeat_interleave(G, dim=1)
    z = torch.matmul(qh, kh.transpose(-1, -2)) * scale
    if bias is not None:
        z = z + bias
    z = z.masked_fill(~mask_bool, float("-inf"))
    return torch.logsumexp(z, dim=-1).transpose(1, 2).numpy()


def all_pred_idx(B, T, q_pos0=0):
    idx = np.full((B, T, q_pos0 + T), -1, dtype=np.int32)
    for t in range(T):
        p = q_pos0 + t
        idx[:, t, :p + 1] = np.arange(p + 1)
    return idx


# ---------------------------------------------------------------- indexer --
def test_indexer_scores_match_numpy_einsum():
    g = torch.Generator().manual_seed(1)
    B, T, L, Hi, di = 2, 37, 53, 3, 16
    q = torch.randint(-8, 9, (B, T, Hi, di), generator=g).to(torch.int8)
    k = torch.randint(-8, 9, (B, L, di), generator=g).to(torch.int8)
    w = torch.randint(0, 5, (B, T, Hi), generator=g).to(torch.int32)
    q_pos0 = L - T
    got = oracle.indexer_scores(q, k, w, q_pos0=q_pos0)
    s = np.einsum("bthc,bjc->bthj", q.numpy().astype(np.int64), k.numpy().astype(np.int64))
    ref = np.einsum("bth,bthj->btj", w.numpy().astype(np.int64), np.maximum(s, 0))
    ref = ref.reshape(B * T, L)
    for r in range(B * T):
        p = q_pos0 + r % T
        np.testing.assert_array_equal(got[r, :p + 1], ref[r, :p + 1])
        assert np.all(got[r, p + 1:] == np.iinfo(np.int64).min)


def test_indexer_negative_weights_follow_formula():
    # w multiplies the ReLU output; a negative weight must subtract.
    q = torch.tensor([[[[2], [1]]]], dtype=torch.int8)   # B=1,T=1,Hi=2,di=1
    k = torch.tensor([[[3], [-3]]], dtype=torch.int8)    # L=2
    w = torch.tensor([[[-1, 5]]], dtype=torch.int32)
    got = oracle.indexer_scores(q, k, w, q_pos0=1)
    # j=0: -1*relu(6) + 5*relu(3) = 9 ; j=1: relu(-6)=0, relu(-3)=0 -> 0
    np.testing.assert_array_equal(got[0], [9, 0])


def _read_topk_golden():
    rows = []
    with open(os.path.join(GOLDEN, "topk_ties.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, exp, _ = line.split("|")
            tk, win = map(int, head.split())
            rows.append((tk, win, [int(x) for x in exp.split()]))
    return rows


@pytest.mark.parametrize("topk,window,expected", _read_topk_golden())
def test_topk_hand_worked_ties(topk, window, expected):
    kv = [3, 1, 3, 0, 2, 3, -1, 3]
    q = torch.ones((1, 1, 1, 1), dtype=torch.int8)
    k = torch.tensor(kv, dtype=torch.int8).reshape(1, 8, 1)
    w = torch.ones((1, 1, 1), dtype=torch.int32)
    idx, cnt = oracle.indexer_topk(q, k, w, topk, window, q_pos0=7)
    got = [int(x) for x in idx[0] if x >= 0]
    assert got == expected
    assert cnt[0] == len(expected)
    assert np.all(idx[0, cnt[0]:] == -1)


def test_topk_brute_force_dominance_tiny():
    d = inputs.gen_dsa(1, 40, 1, 1, 8, 2, 4, seed=3)
    topk, window = 6, 3
    idx, cnt = oracle.indexer_topk(d["q_idx"], d["k_idx"], d["w"], topk, window)
    sc = oracle.indexer_scores(d["q_idx"], d["k_idx"], d["w"])
    for t in range(40):
        sel = set(int(x) for x in idx[t] if x >= 0)
        wset = set(range(max(0, t - window + 1), t + 1))
        assert wset <= sel
        cands = [j for j in range(t + 1) if j not in wset]
        chosen = sel - wset
        assert len(chosen) == min(topk, len(cands))
        assert cnt[t] == len(sel)
        row = list(idx[t][:cnt[t]])
        assert row == sorted(row)
        for a in chosen:
            for b in cands:
                if b in chosen:
                    continue
                # every chosen candidate beats every rejected one
                assert (sc[t, a] > sc[t, b]) or (sc[t, a] == sc[t, b] and a < b)


def test_topk_matches_lexsort_medium():
    d = inputs.gen_dsa(2, 300, 1, 1, 8, 4, 32, seed=5)
    topk = 50
    idx, cnt = oracle.indexer_topk(d["q_idx"], d["k_idx"], d["w"], topk, 0)
    sc = oracle.indexer_scores(d["q_idx"], d["k_idx"], d["w"])
    for r in range(600):
        t = r % 300
        s = sc[r, :t + 1]
        j = np.arange(t + 1)
        order = np.lexsort((j, -s))           # primary: score desc, then j asc
        ref = np.sort(order[:topk])
        np.testing.assert_array_equal(idx[r, :cnt[r]], ref)


def test_topk_window_rule_tiny_workload():
    w = inputs.WORKLOADS["tiny_dsa"]
    d = inputs.gen_dsa(w.B, w.T, w.Hq, w.Hkv, w.d, w.Hi, w.di, seed=0)
    idx, cnt = oracle.indexer_topk(d["q_idx"], d["k_idx"], d["w"], w.topk, w.window)
    for t in range(w.T):
        assert cnt[t] == min(t + 1, w.topk + w.window)
        s = set(idx[t, :cnt[t]].tolist())
        assert set(range(max(0, t - w.window + 1), t + 1)) <= s
        assert max(s) <= t


def test_topk_dense_when_k_covers_all():
    d = inputs.gen_dsa(1, 64, 1, 1, 8, 2, 8, seed=7)
    idx, cnt = oracle.indexer_topk(d["q_idx"], d["k_idx"], d["w"], 64, 0)
    for t in range(64):
        np.testing.assert_array_equal(idx[t, :t + 1], np.arange(t + 1))
        assert cnt[t] == t + 1


# ------------------------------------------------------------ fixed graph --
def _read_graph_golden():
    rows = []
    with open(os.path.join(GOLDEN, "fixed_graph_sets.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, exp, _ = line.split("|")
            win, dil, p = map(int, head.split())
            rows.append((win, dil, p, [int(x) for x in exp.split()]))
    return rows


@pytest.mark.parametrize("window,dilated,p,expected", _read_graph_golden())
def test_fixed_graph_hand_derived(window, dilated, p, expected):
    idx, cnt = oracle.fixed_graph(p + 1, window, bool(dilated), q_pos0=p, Tq=1, cap=80)
    assert idx[0, :cnt[0]].tolist() == expected


def test_fixed_graph_size_closed_form_16k():
    # |S_p| = min(p+1, window) + #{i : window <= 2^i < p}; summed in closed
    # form over i rather than over the oracle's membership scan.
    T, window = 16384, 65
    total = 0
    mx = 0
    for p in range(T):
        n = min(p + 1, window)
        i = 0
        while (1 << i) < p:
            if (1 << i) >= window:
                n += 1
            i += 1
        total += n
        mx = max(mx, n)
    # oracle on a spread of positions, then the full count
    idx, cnt = oracle.fixed_graph(T, window, True, cap=80)
    assert int(cnt.sum()) == total
    assert int(cnt.max()) == mx == 72
    assert np.all(idx[:, 0] >= 0)
    assert np.all((idx < 0) | (idx <= np.arange(T)[:, None]))


# -------------------------------------------------------------- attention --
def test_complete_set_is_dense_causal():
    B, T, Hq, Hkv, d = 2, 48, 4, 1, 32
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 4, seed=11)
    idx = all_pred_idx(B, T)
    out, lse, psum, maxj = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, want_stats=True)
    scale = 1 / math.sqrt(d)
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    ref = sdpa_ref(g["q"], g["k"], g["v"], mask=mask, scale=scale).reshape(B * T, Hq, d)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    lref = lse_ref(g["q"], g["k"], mask, scale).reshape(B * T, Hq)
    np.testing.assert_allclose(lse, lref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(psum, 1.0, atol=1e-12)
    assert np.all(maxj == np.tile(np.arange(T), B))


def test_window_set_is_banded_attention():
    B, T, H, d, W = 1, 70, 2, 16, 9
    g = inputs.gen_dsa(B, T, H, H, d, 1, 4, seed=12)
    idx = np.full((B, T, W), -1, dtype=np.int32)
    for t in range(T):
        lo = max(0, t - W + 1)
        idx[0, t, :t - lo + 1] = np.arange(lo, t + 1)
    out, lse = oracle.sparse_attn(g["q"], g["k"], g["v"], idx)
    i = torch.arange(T)
    mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - W)
    ref = sdpa_ref(g["q"], g["k"], g["v"], mask=mask, scale=1 / math.sqrt(d))
    np.testing.assert_allclose(out, ref.reshape(T, H, d), rtol=0, atol=1e-12)


def test_per_kv_head_lists_and_gqa_mapping():
    # idx_heads == Hkv: KV head g uses its own list; query head h -> h // (Hq/Hkv)
    B, T, Hq, Hkv, d = 1, 20, 4, 2, 8
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 4, seed=13)
    idx = np.full((B, T, Hkv, T), -1, dtype=np.int32)
    for t in range(T):
        idx[0, t, 0, :t + 1] = np.arange(t + 1)        # head group 0: dense
        idx[0, t, 1, 0] = t                            # head group 1: self only
    out, _ = oracle.sparse_attn(g["q"], g["k"], g["v"], idx)
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    ref = sdpa_ref(g["q"], g["k"], g["v"], mask=mask, scale=1 / math.sqrt(d)).reshape(T, Hq, d)
    np.testing.assert_allclose(out[:, :2], ref[:, :2], atol=1e-12)
    vv = g["v"].to(torch.float64).numpy()[0]           # [T, Hkv, d]
    np.testing.assert_allclose(out[:, 2], vv[:, 1], atol=0)
    np.testing.assert_allclose(out[:, 3], vv[:, 1], atol=0)


def test_coordinate_bias_matches_cdist_mask():
    B, T, H, d = 1, 33, 2, 16
    g = inputs.gen_spatial(B, T, H, d, beta=0.7, seed=14)
    g["beta"] = torch.tensor([0.7, 0.2])
    idx = all_pred_idx(B, T)
    out, lse = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, cq=g["cq"], ck=g["ck"],
                                  beta=g["beta"])
    # library distance (cdist) -> additive mask for torch SDPA
    cq = g["cq"].to(torch.float64)[0].transpose(0, 1)     # [H,T,3]
    ck = g["ck"].to(torch.float64)[0].transpose(0, 1)
    dist2 = torch.cdist(cq, ck) ** 2                       # [H,T,T]
    bias = -g["beta"].to(torch.float64)[:, None, None] * dist2
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    mask = bias.masked_fill(~causal, float("-inf"))[None]
    ref = sdpa_ref(g["q"], g["k"], g["v"], mask=mask, scale=1 / math.sqrt(d))
    np.testing.assert_allclose(out, ref.reshape(T, H, d), atol=1e-10)
    lref = lse_ref(g["q"], g["k"], causal, 1 / math.sqrt(d), bias=bias[None])
    np.testing.assert_allclose(lse, lref.reshape(T, H), atol=1e-10)


def test_coordinate_bias_invariances():
    B, T, H, d = 1, 25, 2, 8
    g = inputs.gen_spatial(B, T, H, d, seed=15)
    idx = all_pred_idx(B, T)
    plain, _ = oracle.sparse_attn(g["q"], g["k"], g["v"], idx)
    # beta = 0 -> plain attention
    o0, _ = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, cq=g["cq"], ck=g["ck"],
                               beta=torch.zeros(H))
    np.testing.assert_allclose(o0, plain, atol=1e-14)
    # every key at the same point -> constant bias per row -> plain output
    ck_same = torch.zeros_like(g["ck"]) + 0.25
    o1, _ = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, cq=g["cq"], ck=ck_same,
                               beta=g["beta"])
    np.testing.assert_allclose(o1, plain, atol=1e-12)
    # translating every coordinate leaves distances, hence outputs, unchanged
    shift = torch.tensor([1.5, -2.0, 0.5])
    o2, _ = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, cq=g["cq"], ck=g["ck"],
                               beta=g["beta"])
    o3, _ = oracle.sparse_attn(g["q"], g["k"], g["v"], idx, cq=g["cq"] + shift,
                               ck=g["ck"] + shift, beta=g["beta"])
    np.testing.assert_allclose(o2, o3, atol=1e-5)  # fp32 coordinates re-rounded
    # a nearer key gets more weight: with q = 0 only the bias decides
    q0 = torch.zeros_like(g["q"])
    v_id = torch.zeros_like(g["v"])
    v_id[0, :, :, 0] = torch.arange(T, dtype=torch.float32).to(torch.bfloat16)[:, None]
    cq = torch.zeros_like(g["cq"])
    ck = torch.zeros_like(g["ck"])
    ck[0, 3, :, 0] = 0.0       # key 3 at the query's point, all others far
    ck[0, :3, :, 0] = 5.0
    ck[0, 4:, :, 0] = 5.0
    o4, _ = oracle.sparse_attn(q0, g["k"], v_id, idx, cq=cq, ck=ck, beta=g["beta"])
    assert np.all(np.abs(o4[10:, :, 0] - 3.0) < 1e-3)


def test_empty_list_and_future_index():
    g = inputs.gen_dsa(1, 4, 2, 1, 8, 1, 4, seed=16)
    idx = np.full((1, 4, 3), -1, dtype=np.int32)
    out, lse = oracle.sparse_attn(g["q"], g["k"], g["v"], idx)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    idx[0, 1, 0] = 2          # position 2 is in the future of query 1
    with pytest.raises(oracle.OracleError):
        oracle.sparse_attn(g["q"], g["k"], g["v"], idx)


# ------------------------------------------------------------ lse combine --
def test_lse_combine_equals_unsplit():
    B, T, Hq, d = 1, 60, 4, 16
    g = inputs.gen_dsa(B, T, Hq, 1, d, 1, 4, seed=17)
    idx = all_pred_idx(B, T)
    full, lfull = oracle.sparse_attn(g["q"], g["k"], g["v"], idx)
    for n_split in (2, 3, 7):
        K = idx.shape[-1]
        c = -(-K // n_split)
        po, pl = [], []
        for s in range(n_split):
            part = np.full_like(idx, -1)
            part[..., s * c:(s + 1) * c] = idx[..., s * c:(s + 1) * c]
            o, l = oracle.sparse_attn(g["q"], g["k"], g["v"], part)
            po.append(o.reshape(-1, d))
            pl.append(l.reshape(-1))
        out, lse = oracle.lse_combine(np.stack(po), np.stack(pl))
        np.testing.assert_allclose(out, full.reshape(-1, d), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lfull.reshape(-1), rtol=0, atol=1e-12)


def test_lse_combine_all_empty():
    po = np.random.default_rng(0).standard_normal((3, 5, 4))
    pl = np.full((3, 5), -np.inf)
    out, lse = oracle.lse_combine(po, pl)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ---------------------------------------------------------------- NSA -----
def test_nsa_compress_matches_numpy_means():
    g = inputs.gen_nsa(1, 200, 2, 2, 8, seed=18)
    k64 = g["k"].to(torch.float64).numpy()
    # non-overlapping (stride == len): a reshape mean
    kc, _ = oracle.nsa_compress(g["k"], g["v"], 8, 8)
    ref = k64[:, :200].reshape(1, 25, 8, 2, 8).mean(axis=2)
    np.testing.assert_allclose(kc, ref, atol=1e-14)
    # overlapping (len 32, stride 16): prefix-sum differences
    kc2, vc2 = oracle.nsa_compress(g["k"], g["v"], 32, 16)
    cs = np.concatenate([np.zeros((1, 1, 2, 8)), np.cumsum(k64, axis=1)], axis=1)
    nc = (200 - 32) // 16 + 1
    starts = np.arange(nc) * 16
    ref2 = (cs[:, starts + 32] - cs[:, starts]) / 32
    np.testing.assert_allclose(kc2, ref2, atol=1e-12)
    assert kc2.shape[1] == nc


NSA_SMALL = dict(cmp_len=8, cmp_stride=4, sel_block=16, sel_topk=3, window=12)


def _nsa_small(T=96, Hq=4, Hkv=2, d=16, seed=19):
    g = inputs.gen_nsa(1, T, Hq, Hkv, d, seed=seed)
    r = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], **NSA_SMALL)
    return g, r


def test_nsa_compressed_branch_is_block_causal_sdpa():
    T, d = 96, 16
    g, r = _nsa_small(T=T, d=d)
    L, S = NSA_SMALL["cmp_len"], NSA_SMALL["cmp_stride"]
    kc, vc = oracle.nsa_compress(g["k"], g["v"], L, S)
    nc = kc.shape[1]
    t = torch.arange(T)[:, None]
    i = torch.arange(nc)[None, :]
    vis = (i * S + L - 1) <= t                        # [T, nc]
    rows = vis.any(dim=1).numpy()
    qh = _f64(g["q"]).transpose(1, 2)
    kh = torch.from_numpy(kc).transpose(1, 2)
    vh = torch.from_numpy(vc).transpose(1, 2)
    ref = F.scaled_dot_product_attention(qh[:, :, rows], kh, vh, attn_mask=vis[rows],
                                         scale=1 / math.sqrt(d), enable_gqa=True)
    ref = ref.transpose(1, 2).numpy()[0]
    np.testing.assert_allclose(r["o_branch"][0][rows], ref, atol=1e-12)
    assert np.all(r["o_branch"][0][~rows] == 0)
    assert np.all(np.isneginf(r["lse_branch"][~rows, :, 0]))


def test_nsa_importance_sums_to_group_size():
    # sum over blocks of imp = sum over heads in the group of sum_i p_cmp = G
    T, Hq, Hkv = 96, 4, 2
    g, r = _nsa_small(T=T, Hq=Hq, Hkv=Hkv)
    L = NSA_SMALL["cmp_len"]
    tot = r["imp"].sum(axis=2)                       # [T, Hkv]
    for t in range(T):
        exp = (Hq // Hkv) if t >= L - 1 else 0.0
        np.testing.assert_allclose(tot[t], exp, atol=1e-12)


def test_nsa_selection_dominance_and_format():
    T = 96
    g, r = _nsa_small(T=T)
    sb, k = NSA_SMALL["sel_block"], NSA_SMALL["sel_topk"]
    for t in range(T):
        cands = [b for b in range(r["imp"].shape[2]) if b * sb <= t]
        for gg in range(r["sel_idx"].shape[1]):
            sel = [int(x) for x in r["sel_idx"][t, gg] if x >= 0]
            assert sel == sorted(sel) and len(sel) == min(k, len(cands))
            imp = r["imp"][t, gg]
            for a in sel:
                for b in cands:
                    if b not in sel:
                        assert imp[a] > imp[b] or (imp[a] == imp[b] and a < b)


def test_nsa_selected_branch_dense_when_all_blocks_chosen():
    # t < sel_block * sel_topk: every candidate block is chosen -> dense causal
    T, d = 48, 16      # 3 blocks of 16 == sel_topk
    g = inputs.gen_nsa(1, T, 4, 2, d, seed=20)
    r = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], **NSA_SMALL)
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    ref = sdpa_ref(g["q"], g["k"], g["v"], mask=mask, scale=1 / math.sqrt(d))[0]
    np.testing.assert_allclose(r["o_branch"][1], ref, atol=1e-12)


def test_nsa_window_branch_is_banded():
    T, d, W = 96, 16, NSA_SMALL["window"]
    g, r = _nsa_small(T=T, d=d)
    i = torch.arange(T)
    mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - W)
    ref = sdpa_ref(g["q"], g["k"], g["v"], mask=mask, scale=1 / math.sqrt(d))[0]
    np.testing.assert_allclose(r["o_branch"][2], ref, atol=1e-12)


def test_nsa_gates_isolate_branches():
    T, Hq = 64, 4
    g = inputs.gen_nsa(1, T, Hq, 2, 16, seed=21)
    base = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], **NSA_SMALL)
    # the gated sum of the stored branches reproduces the output
    gates = g["gates"].to(torch.float64).numpy()[0]            # [T,Hq,3]
    comb = np.einsum("thb,bthd->thd", gates, base["o_branch"])
    np.testing.assert_allclose(base["out"], comb, atol=1e-12)
    for br in range(3):
        oh = torch.zeros_like(g["gates"])
        oh[..., br] = 1.0
        r = oracle.nsa_fwd(g["q"], g["k"], g["v"], oh, **NSA_SMALL)
        np.testing.assert_allclose(r["out"], base["o_branch"][br], atol=0)


def test_nsa_planted_block_is_selected():
    # make every query align with the keys of block 2 only: it must be chosen
    T, Hq, Hkv, d = 96, 2, 1, 16
    g = inputs.gen_nsa(1, T, Hq, Hkv, d, seed=22)
    q = torch.zeros_like(g["q"]); q[..., 0] = 4.0
    k = torch.zeros_like(g["k"]); k[0, 32:48, 0, 0] = 4.0
    r = oracle.nsa_fwd(q, k, g["v"], g["gates"], **NSA_SMALL)
    for t in range(48 + NSA_SMALL["cmp_len"], T):
        assert 2 in r["sel_idx"][t, 0].tolist()


def _read_nsa_importance_golden():
    rows = []
    with open(os.path.join(GOLDEN, "nsa_importance.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            ts, imp, sel1, sel3 = [x.strip() for x in line.split("|")]
            t_lo, t_hi = (int(x) for x in ts.split())
            fr = []
            for x in imp.split():
                a, _, b = x.partition("/")
                fr.append(float(a) / float(b or 1))
            rows.append((t_lo, t_hi, fr, [int(x) for x in sel1.split()],
                         [int(x) for x in sel3.split()]))
    return rows


def test_nsa_importance_and_candidates_hand_derived():
    """Block importance (start-position mapping, summed over the group's
    heads) and the candidate rule b*sel_block <= t against the hand-derived
    table in tests/golden/nsa_importance.txt."""
    T, d = 48, 16
    q = torch.zeros(1, T, 2, d, dtype=torch.bfloat16)
    q[0, :, 1, 0] = 16.0
    k = torch.zeros(1, T, 1, d, dtype=torch.bfloat16)
    k[0, 12:20, 0, 0] = 16.0
    v = inputs.gen_nsa(1, T, 2, 1, d, seed=23)["v"]
    gates = torch.full((1, T, 2, 3), 0.5)
    cfg = dict(cmp_len=8, cmp_stride=4, sel_block=16, window=16, scale=1.0)
    r3 = oracle.nsa_fwd(q, k, v, gates, sel_topk=3, **cfg)
    r1 = oracle.nsa_fwd(q, k, v, gates, sel_topk=1, **cfg)
    covered = set()
    for t_lo, t_hi, imp, sel1, sel3 in _read_nsa_importance_golden():
        for t in range(t_lo, t_hi + 1):
            covered.add(t)
            np.testing.assert_allclose(r3["imp"][t, 0], imp, rtol=0, atol=1e-12,
                                       err_msg=f"importance at t={t}")
            assert r1["sel_idx"][t, 0].tolist() == sel1, f"top-1 at t={t}"
            assert r3["sel_idx"][t, 0].tolist() == sel3, f"top-3 at t={t}"
    assert covered == set(range(T))


def test_nsa_override_with_own_selection_is_identity():
    g, r = _nsa_small()
    r2 = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], sel_override=r["sel_idx"],
                        **NSA_SMALL)
    np.testing.assert_array_equal(r2["out"], r["out"])


# ------------------------------------------------------------ IndexCache --
def _decode_layers(n_layers, nseq=2, L=300, seed=23):
    return [inputs.gen_decode_layer(nseq, L, 4, 1, 16, 2, 8, layer=i, seed=seed)
            for i in range(n_layers)]


def test_indexcache_s_layers_reuse_f_indices():
    lays = _decode_layers(4)
    res = oracle.dsa_layers("FSSS", lays, topk=32)
    for i in (1, 2, 3):
        np.testing.assert_array_equal(res[i][0], res[0][0])
        out, lse = oracle.sparse_attn(lays[i]["q"], lays[i]["k"], lays[i]["v"], res[0][0],
                                      q_pos0=299)
        np.testing.assert_array_equal(res[i][1], out)
    allf = oracle.dsa_layers("FFFF", lays, topk=32)
    for i in range(4):
        idx, _ = oracle.indexer_topk(lays[i]["q_idx"], lays[i]["k_idx"], lays[i]["w"], 32,
                                     q_pos0=299)
        np.testing.assert_array_equal(allf[i][0].reshape(idx.shape), idx)


def test_indexcache_pattern_must_start_with_f():
    with pytest.raises(oracle.OracleError):
        oracle.dsa_layers("SFFF", _decode_layers(4), topk=8)


# ------------------------------------------------------- attention backward --
def _autograd_ref(q, k, v, dout, bias, scale):
    """dq, dk, dv of softmax(scale q.k + bias) v by torch float64 autograd;
    bias [B,Hq,T,L] additive (-inf = not in the set).  GQA by repeating the
    KV heads (autograd sums their gradients)."""
    qh = _f64(q).transpose(1, 2).clone().requires_grad_(True)
    kh = _f64(k).transpose(1, 2).clone().requires_grad_(True)
    vh = _f64(v).transpose(1, 2).clone().requires_grad_(True)
    G = qh.shape[1] // kh.shape[1]
    bias = torch.broadcast_to(bias, (qh.shape[0], qh.shape[1], qh.shape[2], kh.shape[2]))
    # a row with an empty set has no gradient: give it a finite bias and no
    # incoming gradient, so softmax stays defined and it contributes nothing
    empty = torch.isneginf(bias).all(dim=-1, keepdim=True)
    bias = torch.where(empty, torch.zeros_like(bias), bias)
    z = torch.matmul(qh, kh.repeat_interleave(G, dim=1).transpose(-1, -2)) * scale + bias
    p = torch.softmax(z, dim=-1)
    o = torch.matmul(p, vh.repeat_interleave(G, dim=1))
    o.backward(_f64(dout).transpose(1, 2).masked_fill(empty, 0.0))
    return (qh.grad.transpose(1, 2).numpy(), kh.grad.transpose(1, 2).numpy(),
            vh.grad.transpose(1, 2).numpy())


def _bias_from_lists(idx, B, Hq, Hkv, T, L):
    """Additive bias log(multiplicity) from index lists [B,T,ih,K]."""
    ii = idx if idx.ndim == 4 else idx[:, :, None, :]
    mult = np.zeros((B, ii.shape[2], T, L))
    for b in range(B):
        for t in range(T):
            for ih in range(ii.shape[2]):
                for j in ii[b, t, ih]:
                    if j >= 0:
                        mult[b, ih, t, j] += 1
    G = Hq // Hkv
    per_head = np.repeat(mult, Hq if ii.shape[2] == 1 else G, axis=1)
    with np.errstate(divide="ignore"):
        return torch.from_numpy(np.log(per_head))


def _bwd_case(B, T, Hq, Hkv, d, seed):
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=seed)
    gen = torch.Generator().manual_seed(seed + 7)
    dout = torch.randn(B, T, Hq, d, generator=gen).to(torch.bfloat16)
    return g["q"], g["k"], g["v"], dout


def test_backward_complete_set_is_dense_causal_autograd():
    B, T, Hq, Hkv, d = 1, 40, 4, 2, 16
    q, k, v, dout = _bwd_case(B, T, Hq, Hkv, d, 70)
    idx = all_pred_idx(B, T)
    dq, dk, dv = oracle.sparse_attn_bwd(q, k, v, dout, idx)
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    bias = torch.zeros(T, T, dtype=torch.float64).masked_fill(~mask, float("-inf"))
    rq, rk, rv = _autograd_ref(q, k, v, dout, bias, 1 / math.sqrt(d))
    np.testing.assert_allclose(dq, rq, atol=1e-10)
    np.testing.assert_allclose(dk, rk, atol=1e-10)
    np.testing.assert_allclose(dv, rv, atol=1e-10)


@pytest.mark.parametrize("idx_heads", [1, 2])
def test_backward_random_lists_with_duplicates(idx_heads):
    # random lists (one shared, or one per KV head), an empty row, a repeated
    # key (a repeat counts twice: bias log 2 in the dense form)
    B, T, Hq, Hkv, d, K = 2, 30, 4, 2, 16, 9
    q, k, v, dout = _bwd_case(B, T, Hq, Hkv, d, 71 + idx_heads)
    rng = np.random.default_rng(5 + idx_heads)
    idx = np.full((B, T, idx_heads, K), -1, dtype=np.int32)
    for b in range(B):
        for t in range(T):
            for ih in range(idx_heads):
                n = min(t + 1, K - 1)
                idx[b, t, ih, :n] = rng.choice(t + 1, size=n, replace=False)
                idx[b, t, ih, K - 1] = idx[b, t, ih, 0]          # duplicate
    idx[1, 5] = -1                                               # empty row
    ii = idx if idx_heads > 1 else idx[:, :, 0, :]
    dq, dk, dv = oracle.sparse_attn_bwd(q, k, v, dout, ii)
    bias = _bias_from_lists(idx, B, Hq, Hkv, T, T)
    rq, rk, rv = _autograd_ref(q, k, v, dout, bias, 1 / math.sqrt(d))
    np.testing.assert_allclose(dq, rq, atol=1e-10)
    np.testing.assert_allclose(dk, rk, atol=1e-10)
    np.testing.assert_allclose(dv, rv, atol=1e-10)
    assert np.all(dq[1, 5] == 0)


def test_backward_column_sum_identities():
    # sum_j dS_j = 0 per (row, head), so sum_j dk_j = 0; sum_j p_j = 1 per
    # non-empty (row, head), so sum_j dv_j = sum of dout over the group's heads
    B, T, Hq, Hkv, d = 1, 64, 8, 2, 32
    q, k, v, dout = _bwd_case(B, T, Hq, Hkv, d, 73)
    rng = np.random.default_rng(9)
    K = 12
    idx = np.full((B, T, K), -1, dtype=np.int32)
    for t in range(T):
        n = min(t + 1, K)
        idx[0, t, :n] = rng.choice(t + 1, size=n, replace=False)
    dq, dk, dv = oracle.sparse_attn_bwd(q, k, v, dout, idx)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-10)
    do = _f64(dout).numpy().reshape(B, T, Hkv, Hq // Hkv, d).sum(axis=(1, 3))
    np.testing.assert_allclose(dv.sum(axis=1), do, atol=1e-10)


# ------------------------------------------------------------ NSA backward --
def _nsa_torch_out(q, k, v, gates, sel, cmp_len, cmp_stride, sel_block, window, scale):
    """NSA forward as dense masked softmaxes in torch float64, with the block
    choice sel [B*T, Hkv, topk] fixed; differentiable in q, k, v, gates.
    Compressed rows come from torch's unfold + mean."""
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    t = torch.arange(T)[:, None]
    branches = []
    # compressed branch over mean-pooled rows
    if T >= cmp_len:
        kc = k.unfold(1, cmp_len, cmp_stride).mean(-1)
        vc = v.unfold(1, cmp_len, cmp_stride).mean(-1)
        i = torch.arange(kc.shape[1])[None, :]
        m = ((i * cmp_stride + cmp_len - 1) <= t)[None, None].expand(B, Hkv, T, kc.shape[1])
        branches.append((kc, vc, m))
    else:
        branches.append(None)
    # selected branch: keys of the chosen blocks, j <= t
    j = torch.arange(T)
    ms = torch.zeros(B, Hkv, T, T, dtype=torch.bool)
    s3 = torch.from_numpy(np.asarray(sel)).reshape(B, T, Hkv, -1)
    for b in range(B):
        for tt in range(T):
            for g in range(Hkv):
                for blk in s3[b, tt, g].tolist():
                    if blk >= 0:
                        ms[b, g, tt] |= (j // sel_block == blk) & (j <= tt)
    branches.append((k, v, ms))
    mw = ((j[None, :] <= t) & (j[None, :] > t - window))[None, None].expand(B, Hkv, T, T)
    branches.append((k, v, mw))
    out = torch.zeros(B, T, Hq, d, dtype=torch.float64)
    for br, item in enumerate(branches):
        if item is None:
            continue
        kk, vv, m = item
        qh = q.transpose(1, 2)                                     # [B,Hq,T,d]
        kh = kk.transpose(1, 2).repeat_interleave(G, dim=1)
        vh = vv.transpose(1, 2).repeat_interleave(G, dim=1)
        mh = m.repeat_interleave(G, dim=1)
        empty = ~mh.any(dim=-1, keepdim=True)
        z = torch.matmul(qh, kh.transpose(-1, -2)) * scale
        z = z.masked_fill(~mh & ~empty, float("-inf"))
        o = torch.matmul(torch.softmax(z, dim=-1), vh).masked_fill(empty, 0.0)
        out = out + gates[..., br:br + 1] * o.transpose(1, 2)
    return out


def _nsa_bwd_case(T, Hq, Hkv, d, seed, cfg):
    g = inputs.gen_nsa(1, T, Hq, Hkv, d, seed=seed)
    gen = torch.Generator().manual_seed(seed + 3)
    dout = torch.randn(1, T, Hq, d, generator=gen).to(torch.bfloat16)
    r = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], **cfg)
    gr = oracle.nsa_bwd(g["q"], g["k"], g["v"], g["gates"], dout, r["sel_idx"], **cfg)
    return g, dout, r, gr


@pytest.mark.parametrize("T,Hq,Hkv,d,cfg", [
    (96, 4, 2, 16, NSA_SMALL),
    (75, 6, 2, 8, dict(cmp_len=8, cmp_stride=4, sel_block=16, sel_topk=2, window=20)),
    (40, 2, 1, 8, dict(cmp_len=16, cmp_stride=8, sel_block=16, sel_topk=4, window=64)),
])
def test_nsa_backward_matches_dense_autograd(T, Hq, Hkv, d, cfg):
    # the hand-written chain rule (per-branch softmax backward, gate factor,
    # compressed-row gradients spread back over the rows they average) against
    # torch autograd of a dense masked formulation of the same forward
    g, dout, r, gr = _nsa_bwd_case(T, Hq, Hkv, d, 31 + T, cfg)
    q = _f64(g["q"]).clone().requires_grad_(True)
    k = _f64(g["k"]).clone().requires_grad_(True)
    v = _f64(g["v"]).clone().requires_grad_(True)
    ga = g["gates"].to(torch.float64).clone().requires_grad_(True)
    out = _nsa_torch_out(q, k, v, ga, r["sel_idx"], cfg["cmp_len"], cfg["cmp_stride"],
                         cfg["sel_block"], cfg["window"], 1 / math.sqrt(d))
    np.testing.assert_allclose(out.detach().numpy()[0], r["out"].reshape(T, Hq, d), atol=1e-12)
    out.backward(_f64(dout))
    np.testing.assert_allclose(gr["dq"], q.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(gr["dk"], k.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(gr["dv"], v.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(gr["dgates"], ga.grad.numpy(), atol=1e-10)


def test_nsa_backward_column_sums():
    # each branch's dS sums to 0 over its keys, and the compressed rows pass
    # their gradient back with weights summing to 1, so sum_j dk_j = 0; each
    # non-empty branch's probabilities sum to 1, so sum_j dv_j is the
    # gate-weighted dout of the group's heads over the live branches
    T, Hq, Hkv, d = 96, 4, 2, 16
    cfg = NSA_SMALL
    g, dout, r, gr = _nsa_bwd_case(T, Hq, Hkv, d, 41, cfg)
    np.testing.assert_allclose(gr["dk"].sum(axis=1), 0.0, atol=1e-10)
    live = np.isfinite(r["lse_branch"])                             # [T,Hq,3]
    w = (g["gates"].numpy()[0].astype(np.float64) * live).sum(axis=-1)   # [T,Hq]
    do = _f64(dout).numpy()[0] * w[..., None]
    expect = do.reshape(T, Hkv, Hq // Hkv, d).sum(axis=(0, 2))
    np.testing.assert_allclose(gr["dv"].sum(axis=1)[0], expect, atol=1e-10)
    # the gate gradient is the upstream gradient against each branch output
    ob = r["o_branch"].reshape(3, T, Hq, d)
    np.testing.assert_allclose(gr["dgates"][0], np.einsum("thc,bthc->thb", _f64(dout).numpy()[0], ob),
                               atol=1e-12)


# ------------------------------------------- full-attention exact indexer --
def _full_case(T=70, Hq=4, Hkv=2, d=16, seed=61):
    g = inputs.gen_dsa(1, T, Hq, Hkv, d, 1, 32, seed=seed)
    return g["q"], g["k"], g["v"]


def _select_ref(scores, T, topk, window):
    """Window + top-k of the rest by (score desc, index asc) with numpy lexsort."""
    K = topk + window
    idx = np.full((T, K), -1, dtype=np.int32)
    for t in range(T):
        w_lo = max(0, t - window + 1) if window > 0 else t + 1
        j = np.arange(w_lo)
        order = np.lexsort((j, -scores[t, :w_lo]))
        chosen = np.sort(np.concatenate([j[order[:topk]], np.arange(w_lo, t + 1)]))
        idx[t, :len(chosen)] = chosen
    return idx


def test_full_attn_indexer_layer_is_causal_sdpa():
    T, Hq, Hkv, d = 70, 4, 2, 16
    q, k, v = _full_case(T, Hq, Hkv, d)
    out, lse, idx, sc = oracle.full_attn_topk(q, k, v, topk=8, window=4, want_scores=True)
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    np.testing.assert_allclose(out, sdpa_ref(q, k, v, mask=mask, scale=1 / math.sqrt(d))[0], atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref(q, k, mask, 1 / math.sqrt(d))[0], atol=1e-12)


def test_full_attn_indexer_scores_are_head_summed_probabilities():
    # torch softmax of the masked logits, summed over the heads; every row
    # sums to Hq (each head's probabilities sum to one)
    T, Hq, Hkv, d = 70, 4, 2, 16
    q, k, v = _full_case(T, Hq, Hkv, d)
    _, _, _, sc = oracle.full_attn_topk(q, k, v, topk=8, window=4, want_scores=True)
    qh = _f64(q).transpose(1, 2)
    kh = _f64(k).transpose(1, 2).repeat_interleave(Hq // Hkv, dim=1)
    z = torch.matmul(qh, kh.transpose(-1, -2)) / math.sqrt(d)
    z = z.masked_fill(~torch.ones(T, T, dtype=torch.bool).tril(), float("-inf"))
    ref = torch.softmax(z, dim=-1).sum(dim=1)[0].numpy()
    np.testing.assert_allclose(sc, ref, atol=1e-12)
    np.testing.assert_allclose(sc.sum(axis=1), Hq, atol=1e-12)


@pytest.mark.parametrize("topk,window", [(8, 4), (5, 0), (30, 40), (1, 1)])
def test_full_attn_indexer_selection_matches_lexsort(topk, window):
    T, Hq, Hkv, d = 70, 4, 2, 16
    q, k, v = _full_case(T, Hq, Hkv, d)
    k = k.clone()
    k[0, 20] = k[0, 10]          # duplicated keys: exactly equal scores, lower index first
    k[0, 33] = k[0, 10]
    _, _, idx, sc = oracle.full_attn_topk(q, k, v, topk=topk, window=window, want_scores=True)
    assert np.all(sc[:, 10][34:] == sc[:, 20][34:]) and np.all(sc[:, 20][34:] == sc[:, 33][34:])
    np.testing.assert_array_equal(idx, _select_ref(sc, T, topk, window))


def test_full_attn_indexer_picks_planted_key():
    # a key that every head's query points at collects most of each row's
    # probability and is chosen by every later query
    T, Hq, Hkv, d = 64, 4, 1, 16
    q, k, v = _full_case(T, Hq, Hkv, d, seed=62)
    q = q.clone()
    k = k.clone()
    direction = torch.zeros(d)
    direction[3] = 1.0
    k[0, 7, 0] = (direction * 8).to(torch.bfloat16)
    q[0, :, :] = (q[0, :, :].float() * 0.1 + direction * 4).to(torch.bfloat16)
    _, _, idx = oracle.full_attn_topk(q, k, v, topk=2, window=2)
    for t in range(10, T):
        assert 7 in idx[t]
