"""GPU parity of the sparse-attention backward (sa_sparse_attn_bwd) against
the fp64 oracle: dq, dk and dv over random index lists, per-KV-head lists,
empty rows and repeated entries, and the complete causal set; at a larger
size, identities that hold for any input (sum_j dk_j = 0, sum_j dv_j =
sum of dout over the group's heads).

Tolerance.  The kernel rounds P and dS to bf16 for its tensor-core products
and takes D = dout . out from the forward's bf16 out; each rounding moves a
term by at most 2^-9 relative, so an element is checked to within
2^-6 * max|ref| (max-abs) and 2^-8 * mean|ref| (mean-abs) of the fp64
gradient."""
import math

import numpy as np
import pytest
import torch

import oracle
from fixed_pattern_sparse_sa_b200 import api, inputs
from _parity import sample_rows

pytestmark = pytest.mark.gpu

MAX_REL = 2.0 ** -6
MEAN_REL = 2.0 ** -8


def _close(got, ref, what):
    g = got.detach().double().cpu().numpy().reshape(ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    err = np.abs(g - ref)
    scale_max, scale_mean = np.abs(ref).max(), np.abs(ref).mean()
    assert err.max() <= MAX_REL * scale_max + 1e-6, f"{what}: max err {err.max():.3e} vs {scale_max:.3e}"
    assert err.mean() <= MEAN_REL * scale_mean + 1e-7, f"{what}: mean err {err.mean():.3e} vs {scale_mean:.3e}"


def _lists(B, T, ih, K, seed, dup=False):
    rng = np.random.default_rng(seed)
    idx = np.full((B, T, ih, K), -1, dtype=np.int32)
    for b in range(B):
        for t in range(T):
            for h in range(ih):
                n = min(t + 1, K - (1 if dup else 0))
                idx[b, t, h, :n] = rng.choice(t + 1, size=n, replace=False)
                if dup:
                    idx[b, t, h, K - 1] = idx[b, t, h, 0]
    return torch.from_numpy(idx)


def _run(q, k, v, idx, dout):
    out, lse = api.sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), idx.cuda())
    dq, dk, dv = api.sparse_attn_bwd(q.cuda(), k.cuda(), v.cuda(), out, lse, dout.cuda(), idx.cuda())
    api.check_device_status()
    return dq, dk, dv


@pytest.mark.parametrize("B,T,Hq,Hkv,d,K,ih,dup", [
    (1, 300, 16, 1, 128, 200, 1, False),     # MQA group of 16, lists shorter than the row
    (2, 257, 8, 2, 64, 90, 2, True),         # per-KV-head lists, repeats, ragged chunks
    (1, 129, 12, 1, 128, 64, 1, True),       # 12 heads (a partial m16 tile)
])
def test_backward_random_lists(cuda_ok, B, T, Hq, Hkv, d, K, ih, dup):
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=T + d)
    gen = torch.Generator().manual_seed(T)
    dout = torch.randn(B, T, Hq, d, generator=gen).to(torch.bfloat16)
    idx = _lists(B, T, ih, K, seed=T, dup=dup)
    if ih == 1:
        idx = idx[:, :, 0]
    idx[0, 3] = -1                                       # an empty row
    dq, dk, dv = _run(g["q"], g["k"], g["v"], idx, dout)
    rq, rk, rv = oracle.sparse_attn_bwd(g["q"], g["k"], g["v"], dout, idx)
    _close(dq, rq, "dq")
    _close(dk, rk, "dk")
    _close(dv, rv, "dv")
    assert torch.count_nonzero(dq[0, 3]) == 0


def test_backward_complete_causal_set(cuda_ok):
    B, T, Hq, Hkv, d = 1, 200, 16, 1, 128
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=5)
    dout = torch.randn(B, T, Hq, d, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    idx = torch.full((B, T, T), -1, dtype=torch.int32)
    for t in range(T):
        idx[0, t, :t + 1] = torch.arange(t + 1)
    dq, dk, dv = _run(g["q"], g["k"], g["v"], idx, dout)
    rq, rk, rv = oracle.sparse_attn_bwd(g["q"], g["k"], g["v"], dout, idx)
    _close(dq, rq, "dq")
    _close(dk, rk, "dk")
    _close(dv, rv, "dv")


def test_backward_identities_16k(cuda_ok):
    # 16384 queries x top-512 random lists: sum_j dk_j = 0 and
    # sum_j dv_j = sum over (t, heads of the group) of dout; dq on sampled rows
    B, T, Hq, Hkv, d, K = 1, 16384, 16, 1, 128, 512
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=11)
    dout = torch.randn(B, T, Hq, d, generator=torch.Generator().manual_seed(12)).to(torch.bfloat16)
    dev = torch.device("cuda")
    t = torch.arange(T)
    r = torch.rand(T, K, generator=torch.Generator().manual_seed(13))    # seeded input lists, drawn on the host
    idx = torch.minimum((r * (t[:, None] + 1).float()).long(), t[:, None]).to(torch.int32)[None].to(dev)
    dq, dk, dv = _run(g["q"], g["k"], g["v"], idx, dout)
    sk = dk.double().sum(dim=1).cpu().numpy()
    assert np.abs(sk).max() <= MAX_REL * dk.abs().sum(dim=1).max().item()
    sv = dv.double().sum(dim=1).cpu().numpy()
    ref = dout.double().sum(dim=(1, 2)).numpy()[:, None, :]
    np.testing.assert_allclose(sv, ref, rtol=0, atol=MAX_REL * np.abs(ref).max() + 1e-3)
    # dq of sampled rows from the oracle (its dk / dv need every row); the
    # bound is relative to the gradient's scale over the sampled rows
    rows = sample_rows(T, 8, seed=2, edge=2)
    got, ref = [], []
    for row in rows:
        one = idx.cpu()[:, row:row + 1]
        qq, dd = g["q"][:, row:row + 1], dout[:, row:row + 1]
        rqi, _, _ = oracle.sparse_attn_bwd(qq, g["k"][:, :row + 1], g["v"][:, :row + 1], dd, one, q_pos0=row)
        got.append(dq[:, row:row + 1].double().cpu())
        ref.append(rqi)
    _close(torch.cat(got, dim=1), np.concatenate(ref, axis=1), "dq (sampled rows)")


# ------------------------------------------------------------ NSA backward --
# Tolerance as above: P and dS are rounded to bf16 for the tensor-core
# products, the compressed keys are a bf16 hi/lo pair and the compressed
# values are rounded once to bf16 (as in the forward).  The block choice is
# the forward's; the oracle makes its own and the test requires the two to
# agree, so both sides differentiate the same function.
def _nsa_bwd_gpu(g, dout, cfg):
    dev = "cuda"
    q, k, v, gates = (g[n].to(dev) for n in ("q", "k", "v", "gates"))
    out, lse3, sel, o3 = api.nsa_fwd_train(q, k, v, gates, **cfg)
    dq, dk, dv, dg = api.nsa_bwd(q, k, v, gates, dout.to(dev), o3, lse3, sel, **cfg)
    api.check_device_status()
    return out, sel, dq, dk, dv, dg


@pytest.mark.parametrize("T,Hq,Hkv,d,cfg", [
    # tcgen05 forward path (d = 128, group of 16), real selection
    (640, 32, 2, 128, dict(cmp_len=32, cmp_stride=16, sel_block=64, sel_topk=4, window=128)),
    # d = 64, ragged T, selection blocks not a power of two apart from the window
    (333, 8, 2, 64, dict(cmp_len=16, cmp_stride=8, sel_block=32, sel_topk=3, window=50)),
    # 12 heads per KV head, every candidate block chosen, window longer than T
    (200, 12, 1, 128, dict(cmp_len=32, cmp_stride=16, sel_block=64, sel_topk=16, window=512)),
    # T shorter than one compressed window: the compressed branch is empty
    (20, 4, 1, 64, dict(cmp_len=32, cmp_stride=16, sel_block=16, sel_topk=2, window=8)),
    # the same at head dim 128 (the tcgen05 dq pass writes dq with no key tile)
    (21, 16, 1, 128, dict(cmp_len=32, cmp_stride=16, sel_block=16, sel_topk=2, window=8)),
    # the 64K workload's branch settings on a ragged 2065-token sequence: several
    # 256 / 512-query splits per key block, block lists longer than one work item
    (2065, 16, 1, 128, dict(cmp_len=32, cmp_stride=16, sel_block=64, sel_topk=16, window=512)),
])
def test_nsa_backward_parity(cuda_ok, T, Hq, Hkv, d, cfg):
    g = inputs.gen_nsa(1, T, Hq, Hkv, d, seed=100 + T)
    gen = torch.Generator().manual_seed(200 + T)
    dout = torch.randn(1, T, Hq, d, generator=gen).to(torch.bfloat16)
    ref_f = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], **cfg)
    ref = oracle.nsa_bwd(g["q"], g["k"], g["v"], g["gates"], dout, ref_f["sel_idx"], **cfg)
    out, sel, dq, dk, dv, dg = _nsa_bwd_gpu(g, dout, cfg)
    assert np.array_equal(sel.cpu().numpy().reshape(ref_f["sel_idx"].shape), ref_f["sel_idx"])
    _close(dq, ref["dq"], "dq")
    _close(dk, ref["dk"], "dk")
    _close(dv, ref["dv"], "dv")
    _close(dg, ref["dgates"], "dgates")


def test_nsa_backward_two_sequences(cuda_ok):
    # two sequences in one call: batch offsets of every kernel (the tcgen05
    # dq and key-major passes, the inverse block lists, the pooling backward)
    B, T, Hq, Hkv, d = 2, 420, 16, 2, 128
    cfg = dict(cmp_len=32, cmp_stride=16, sel_block=64, sel_topk=3, window=96)
    g = inputs.gen_nsa(B, T, Hq, Hkv, d, seed=77)
    gen = torch.Generator().manual_seed(78)
    dout = torch.randn(B, T, Hq, d, generator=gen).to(torch.bfloat16)
    ref_f = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], **cfg)
    ref = oracle.nsa_bwd(g["q"], g["k"], g["v"], g["gates"], dout, ref_f["sel_idx"], **cfg)
    out, sel, dq, dk, dv, dg = _nsa_bwd_gpu(g, dout, cfg)
    assert np.array_equal(sel.cpu().numpy().reshape(ref_f["sel_idx"].shape), ref_f["sel_idx"])
    _close(dq, ref["dq"], "dq")
    _close(dk, ref["dk"], "dk")
    _close(dv, ref["dv"], "dv")
    _close(dg, ref["dgates"], "dgates")


@pytest.mark.parametrize("T", [8192, 65536])
def test_nsa_backward_identities(cuda_ok, T):
    # any input: sum_j dk_j = 0 per KV head; sum_j dv_j = the gate-weighted
    # dout of the group's heads over the branches that see at least one key.
    # 65536 tokens is the benchmark's NSA workload and launch configuration.
    Hq, Hkv, d = 64, 4, 128
    cfg = dict(cmp_len=32, cmp_stride=16, sel_block=64, sel_topk=16, window=512)
    g = inputs.gen_nsa(1, T, Hq, Hkv, d, seed=7)
    gen = torch.Generator().manual_seed(8)
    dout = torch.randn(1, T, Hq, d, generator=gen).to(torch.bfloat16)
    out, sel, dq, dk, dv, dg = _nsa_bwd_gpu(g, dout, cfg)
    # the sums in fp64 on the device (the 65536-token tensors are large on the host)
    dk64, dv64 = dk.double(), dv.double()
    live = torch.ones(T, Hq, 3, dtype=torch.float64, device="cuda")
    live[: cfg["cmp_len"] - 1, :, 0] = 0.0                 # no compressed row visible yet
    w = (g["gates"][0].cuda().double() * live).sum(-1)      # [T, Hq]
    expect = (dout[0].cuda().double() * w[..., None]).reshape(T, Hkv, Hq // Hkv, d).sum(dim=(0, 2))
    scale = dv64.abs().sum(dim=1)[0]                        # [Hkv, d]
    assert torch.all((dv64.sum(dim=1)[0] - expect).abs() <= 1e-3 * scale + 1e-3)
    assert torch.all(dk64.sum(dim=1)[0].abs() <= 1e-3 * dk64.abs().sum(dim=1)[0] + 1e-3)
    # the gate gradient against the oracle's branch outputs on sampled rows
    # (the selected branch's only where the block choice equals the oracle's)
    rows = np.array([0, 31, 32, 1000, 4097, T // 2 + 5, T - 1])
    ref_f = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], **cfg, rows=rows)
    dgr = np.einsum("rhc,brhc->rhb", dout[0][torch.from_numpy(rows)].double().numpy(),
                    ref_f["o_branch"].reshape(3, len(rows), Hq, d))
    same = np.all(np.sort(sel[0].cpu().numpy()[rows].reshape(len(rows), -1), axis=1)
                  == np.sort(ref_f["sel_idx"].reshape(len(rows), -1), axis=1), axis=1)
    got = dg[0].cpu()[rows]
    _close(got[..., [0, 2]], dgr[..., [0, 2]], "dgates of the compressed and window branches (sampled rows)")
    if same.any():
        keep = np.nonzero(same)[0]
        _close(got[keep][..., 1], dgr[keep][..., 1], "dgates of the selected branch (sampled rows)")


def test_nsa_backward_bad_block_sets_error_word(cuda_ok):
    # a selected block past the sequence is skipped and reported through the
    # device error word (status 5); the word is cleared by the check
    from fixed_pattern_sparse_sa_b200._lib import SAError
    T, Hq, Hkv, d = 128, 4, 1, 64
    cfg = dict(cmp_len=16, cmp_stride=8, sel_block=16, sel_topk=2, window=16)
    g = inputs.gen_nsa(1, T, Hq, Hkv, d, seed=5)
    q, k, v, gates = (g[n].cuda() for n in ("q", "k", "v", "gates"))
    out, lse3, sel, o3 = api.nsa_fwd_train(q, k, v, gates, **cfg)
    api.check_device_status()
    sel[0, 50, 0, 0] = 1000
    dout = torch.randn(1, T, Hq, d, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).cuda()
    api.nsa_bwd(q, k, v, gates, dout, o3, lse3, sel, **cfg)
    with pytest.raises(SAError) as ei:
        api.check_device_status()
    assert ei.value.status == 5
    api.check_device_status()
