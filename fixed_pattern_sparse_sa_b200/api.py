"""Thin torch binding over libsa.so.

Argument marshalling only: every function checks dtypes, devices and
contiguity, allocates outputs and workspace with torch, and calls the C entry
point of the same name on the current CUDA stream.  All computation happens in
the library's kernels; there is no CPU path.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import SAError, check, sa_dsa_layer, sa_pattern

__all__ = ["indexer_topk", "sparse_attn_fwd", "sparse_attn_bwd", "sparse_attn_fwd_split_static", "lse_combine",
           "nsa_fwd", "indexer_scores_at", "topk_merge", "index_shard",
           "dsa_decode_layers", "check_device_status", "debug_set_spin_limit", "debug_inject_stall",
           "debug_exact_recompute_rows", "SAError"]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: Optional[torch.Tensor], name: str, dtype, dev=None, ndim=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dev is not None and t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _workspace(nbytes: int, device) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def check_device_status(device=None):
    """Wait for the current stream and raise if a kernel found a bad index
    (SA_ERR_DEVICE_ASSERT) or stopped on a bounded wait (SA_ERR_TIMEOUT)."""
    lib = _lib.load()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        check(lib.sa_check_device_status(_stream(None)), "sa_check_device_status")


def debug_set_spin_limit(cycles: int, device=None):
    """sa_debug_set_spin_limit: SM clocks a kernel's progress wait may spin
    before it reports SA_ERR_TIMEOUT; cycles <= 0 restores the default."""
    lib = _lib.load()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        check(lib.sa_debug_set_spin_limit(int(cycles)), "sa_debug_set_spin_limit")


def debug_inject_stall(on: bool, device=None):
    """sa_debug_inject_stall: make the NSA tensor-core branch kernels wait on
    a barrier that nothing completes (a test of the timeout path)."""
    lib = _lib.load()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        check(lib.sa_debug_inject_stall(1 if on else 0), "sa_debug_inject_stall")


def debug_exact_recompute_rows(device=None) -> int:
    """sa_debug_exact_recompute_rows: rows whose top-k was taken by exact
    recompute since the last call (synchronizes the device)."""
    lib = _lib.load()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        n = int(lib.sa_debug_exact_recompute_rows())
    if n < 0:
        check(-n, "sa_debug_exact_recompute_rows")
    return n


# ------------------------------------------------------------------ indexer --
def indexer_topk(q_idx, k_idx, w, topk: int, window: int = 0,
                 q_pos0: Optional[int] = None, out_idx=None, out_count=None, workspace=None):
    """Exact causal top-k of the lightweight indexer (sa_indexer_topk).

    q_idx int8 [B,Tq,Hi,di], k_idx int8 [B,L,di], w int32 [B,Tq,Hi].
    q_pos0 defaults to L - Tq (the queries are the last Tq positions).
    Returns (idx int32 [B,Tq,topk+window], count int32 [B,Tq]).
    """
    lib = _lib.load()
    dev = q_idx.device
    _need(q_idx, "q_idx", torch.int8, dev, 4)
    _need(k_idx, "k_idx", torch.int8, dev, 3)
    _need(w, "w", torch.int32, dev, 3)
    B, Tq, Hi, di = q_idx.shape
    L = k_idx.shape[1]
    if k_idx.shape != (B, L, di) or w.shape != (B, Tq, Hi):
        raise ValueError("indexer_topk: shape mismatch")
    pos0 = L - Tq if q_pos0 is None else int(q_pos0)
    K = topk + window
    if out_idx is None:
        out_idx = torch.empty((B, Tq, K), dtype=torch.int32, device=dev)
    if out_count is None:
        out_count = torch.empty((B, Tq), dtype=torch.int32, device=dev)
    nbytes = lib.sa_indexer_topk_workspace_size(B, Tq, L, Hi, di, topk, window)
    ws = workspace if (workspace is not None and workspace.numel() >= nbytes) \
        else _workspace(nbytes, dev)
    with torch.cuda.device(dev):
        check(lib.sa_indexer_topk(_ptr(q_idx), _ptr(k_idx), _ptr(w), B, Tq, L, Hi, di, pos0,
                                  topk, window, _ptr(out_idx), _ptr(out_count), _ptr(ws),
                                  nbytes, _stream(dev)), "sa_indexer_topk")
    return out_idx, out_count


# ---------------------------------------------------------------- attention --
def sparse_attn_fwd(q, k, v, idx=None, pattern: Optional[Sequence[int]] = None,
                    cq=None, ck=None, beta=None, scale: Optional[float] = None,
                    n_split: int = 1, q_pos0: Optional[int] = None,
                    return_partials: bool = False, out=None, lse=None):
    """Gathered-KV sparse attention (sa_sparse_attn_fwd).

    q bf16 [B,Tq,Hq,d], k/v bf16 [B,L,Hkv,d]; idx int32 [B,Tq,K] or
    [B,Tq,idx_heads,K] (-1 padded), or pattern = (window, dilated).
    Optional coordinate bias cq fp32 [B,Tq,Hq,3], ck fp32 [B,L,Hkv,3],
    beta fp32 [Hq].  Returns (out bf16 [B,Tq,Hq,d], lse fp32 [B,Tq,Hq]) and,
    with return_partials (n_split > 1), also (part_o, part_lse).
    """
    lib = _lib.load()
    dev = q.device
    _need(q, "q", torch.bfloat16, dev, 4)
    _need(k, "k", torch.bfloat16, dev, 4)
    _need(v, "v", torch.bfloat16, dev, 4)
    B, Tq, Hq, d = q.shape
    L, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, L, Hkv, d) or v.shape != k.shape:
        raise ValueError("sparse_attn_fwd: k/v shape mismatch")
    pos0 = L - Tq if q_pos0 is None else int(q_pos0)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    pat = None
    idx_heads, K = 1, 0
    if idx is not None:
        _need(idx, "idx", torch.int32, dev)
        if idx.dim() == 3:
            idx_heads, K = 1, idx.shape[2]
        elif idx.dim() == 4:
            idx_heads, K = idx.shape[2], idx.shape[3]
        else:
            raise ValueError("idx must be [B,Tq,K] or [B,Tq,idx_heads,K]")
        if idx.shape[:2] != (B, Tq):
            raise ValueError("idx shape mismatch")
    elif pattern is not None:
        pat = sa_pattern(int(pattern[0]), int(bool(pattern[1])))
    else:
        raise ValueError("need idx or pattern")
    if cq is not None or ck is not None or beta is not None:
        _need(cq, "cq", torch.float32, dev, 4)
        _need(ck, "ck", torch.float32, dev, 4)
        _need(beta, "beta", torch.float32, dev, 1)
    if out is None:
        out = torch.empty((B, Tq, Hq, d), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=dev)
    po = pl = None
    if n_split > 1:
        po = torch.empty((n_split, B, Tq, Hq, d), dtype=torch.float32, device=dev)
        pl = torch.empty((n_split, B, Tq, Hq), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        check(lib.sa_sparse_attn_fwd(
            _ptr(q), _ptr(k), _ptr(v), B, Tq, L, Hq, Hkv, d, pos0,
            _ptr(idx), idx_heads, K, ctypes.byref(pat) if pat is not None else None,
            _ptr(cq), _ptr(ck), _ptr(beta), float(scale), int(n_split),
            _ptr(out), _ptr(lse), _ptr(po), _ptr(pl), None, 0, _stream(dev)),
            "sa_sparse_attn_fwd")
    if return_partials:
        return out, lse, po, pl
    return out, lse


def sparse_attn_fwd_split_static(q, k, v, idx, n_split: int, scale: Optional[float] = None,
                                 q_pos0: Optional[int] = None, out=None, lse=None):
    """Split-KV sparse attention over index lists that allocates no device
    memory (sa_sparse_attn_fwd_split_static).

    For callers that cannot allocate at call time; the partial results live in
    a fixed 8 MiB array inside the library, so n_split*B*Tq*Hq*(d+1)*4 bytes
    must fit in it, and calls that may overlap on the GPU must be ordered by
    the caller.  Pass out/lse to allocate nothing here either.
    """
    lib = _lib.load()
    dev = q.device
    _need(q, "q", torch.bfloat16, dev, 4)
    _need(k, "k", torch.bfloat16, dev, 4)
    _need(v, "v", torch.bfloat16, dev, 4)
    _need(idx, "idx", torch.int32, dev)
    B, Tq, Hq, d = q.shape
    L, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, L, Hkv, d) or v.shape != k.shape:
        raise ValueError("sparse_attn_fwd_split_static: k/v shape mismatch")
    if idx.dim() == 3:
        idx_heads, K = 1, idx.shape[2]
    elif idx.dim() == 4:
        idx_heads, K = idx.shape[2], idx.shape[3]
    else:
        raise ValueError("idx must be [B,Tq,K] or [B,Tq,idx_heads,K]")
    pos0 = L - Tq if q_pos0 is None else int(q_pos0)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Tq, Hq, d), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        check(lib.sa_sparse_attn_fwd_split_static(
            _ptr(q), _ptr(k), _ptr(v), B, Tq, L, Hq, Hkv, d, pos0, _ptr(idx), idx_heads, K,
            float(scale), int(n_split), _ptr(out), _ptr(lse), _stream(dev)),
            "sa_sparse_attn_fwd_split_static")
    return out, lse


def sparse_attn_bwd(q, k, v, out, lse, dout, idx, scale: Optional[float] = None,
                    q_pos0: Optional[int] = None):
    """Backward of sparse_attn_fwd over explicit index lists (sa_sparse_attn_bwd).

    q, out, dout bf16 [B,Tq,Hq,d]; k, v bf16 [B,L,Hkv,d]; lse fp32 [B,Tq,Hq]
    (the forward's); idx int32 [B,Tq,K] or [B,Tq,idx_heads,K].
    Returns (dq fp32 [B,Tq,Hq,d], dk fp32 [B,L,Hkv,d], dv fp32 [B,L,Hkv,d]).
    """
    lib = _lib.load()
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, n, torch.bfloat16, dev, 4)
    _need(lse, "lse", torch.float32, dev, 3)
    _need(idx, "idx", torch.int32, dev)
    B, Tq, Hq, d = q.shape
    L, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, L, Hkv, d) or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("sparse_attn_bwd: shape mismatch")
    idx_heads = 1 if idx.dim() == 3 else idx.shape[2]
    K = idx.shape[-1]
    pos0 = L - Tq if q_pos0 is None else int(q_pos0)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty((B, Tq, Hq, d), dtype=torch.float32, device=dev)
    dk = torch.empty((B, L, Hkv, d), dtype=torch.float32, device=dev)
    dv = torch.empty((B, L, Hkv, d), dtype=torch.float32, device=dev)
    nbytes = lib.sa_sparse_attn_bwd_workspace_size(B, Tq, Hq)
    ws = _workspace(nbytes, dev)
    with torch.cuda.device(dev):
        check(lib.sa_sparse_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                                     B, Tq, L, Hq, Hkv, d, pos0, _ptr(idx), idx_heads, K, float(scale),
                                     _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), nbytes, _stream(dev)),
              "sa_sparse_attn_bwd")
    return dq, dk, dv


def indexer_scores_at(q_idx, k_idx, w, idx):
    """Exact indexer scores of listed keys (sa_indexer_scores_at).

    q_idx int8 [B,Tq,Hi,di], k_idx int8 [B,L,di], w int32 [B,Tq,Hi],
    idx int32 [B,Tq,K] (-1 = none).  Returns int32 [B,Tq,K] (INT_MIN for -1).
    """
    lib = _lib.load()
    dev = q_idx.device
    _need(q_idx, "q_idx", torch.int8, dev, 4)
    _need(k_idx, "k_idx", torch.int8, dev, 3)
    _need(w, "w", torch.int32, dev, 3)
    _need(idx, "idx", torch.int32, dev, 3)
    B, Tq, Hi, di = q_idx.shape
    out = torch.empty(idx.shape, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        check(lib.sa_indexer_scores_at(_ptr(q_idx), _ptr(k_idx), _ptr(w), B, Tq, k_idx.shape[1], Hi, di,
                                       _ptr(idx), idx.shape[-1], _ptr(out), _stream(dev)), "sa_indexer_scores_at")
    return out


def topk_merge(cand_score, cand_idx, part_off, topk: int, window: int, q_pos: int):
    """Exact top-k of gathered candidates (sa_topk_merge).

    cand_score / cand_idx int32 [n_parts, rows, kc] (part-local indices, -1 =
    none); part_off: n_parts ints (position of each part's index 0).  Returns
    (idx int32 [rows, topk+window] ascending, -1 padded, count int32 [rows]).
    """
    lib = _lib.load()
    dev = cand_score.device
    _need(cand_score, "cand_score", torch.int32, dev, 3)
    _need(cand_idx, "cand_idx", torch.int32, dev, 3)
    n_parts, rows, kc = cand_score.shape
    offs = (ctypes.c_int64 * n_parts)(*[int(x) for x in part_off])
    out = torch.empty((rows, topk + window), dtype=torch.int32, device=dev)
    cnt = torch.empty((rows,), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        check(lib.sa_topk_merge(_ptr(cand_score), _ptr(cand_idx), offs, n_parts, rows, kc, topk, window,
                                int(q_pos), _ptr(out), _ptr(cnt), _stream(dev)), "sa_topk_merge")
    return out, cnt


def index_shard(idx, key_lo: int, key_hi: int):
    """Positions -> rows of the shard [key_lo, key_hi), -1 elsewhere (sa_index_shard)."""
    lib = _lib.load()
    dev = idx.device
    _need(idx, "idx", torch.int32, dev)
    out = torch.empty_like(idx)
    with torch.cuda.device(dev):
        check(lib.sa_index_shard(_ptr(idx), idx.numel(), int(key_lo), int(key_hi), _ptr(out), _stream(dev)),
              "sa_index_shard")
    return out


def lse_combine(part_o, part_lse, out=None, lse=None):
    """Log-sum-exp merge of split partials (sa_lse_combine).

    part_o fp32 [S, ..., d], part_lse fp32 [S, ...] -> (out bf16 [..., d], lse fp32 [...]).
    """
    lib = _lib.load()
    dev = part_o.device
    _need(part_o, "part_o", torch.float32, dev)
    _need(part_lse, "part_lse", torch.float32, dev)
    S, d = part_o.shape[0], part_o.shape[-1]
    lead = tuple(part_o.shape[1:-1])
    if tuple(part_lse.shape) != (S, *lead):
        raise ValueError("lse_combine: shape mismatch")
    rows = math.prod(lead)
    if out is None:
        out = torch.empty((*lead, d), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(lead, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        check(lib.sa_lse_combine(_ptr(part_o), _ptr(part_lse), S, rows, d, _ptr(out), _ptr(lse),
                                 _stream(dev)), "sa_lse_combine")
    return out, lse


# ---------------------------------------------------------------------- NSA --
def nsa_fwd(q, k, v, gates, cmp_len: int, cmp_stride: int, sel_block: int, sel_topk: int,
            window: int, scale: Optional[float] = None, out=None):
    """NSA forward (sa_nsa_fwd): compressed, selected and window branches.

    Returns (out bf16 [B,T,Hq,d], lse_branches fp32 [B,T,Hq,3],
    sel_idx int32 [B,T,Hkv,sel_topk]).
    """
    lib = _lib.load()
    dev = q.device
    _need(q, "q", torch.bfloat16, dev, 4)
    _need(k, "k", torch.bfloat16, dev, 4)
    _need(v, "v", torch.bfloat16, dev, 4)
    _need(gates, "gates", torch.float32, dev, 4)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, d) or v.shape != k.shape or gates.shape != (B, T, Hq, 3):
        raise ValueError("nsa_fwd: shape mismatch")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device=dev)
    lse3 = torch.empty((B, T, Hq, 3), dtype=torch.float32, device=dev)
    sel = torch.empty((B, T, Hkv, sel_topk), dtype=torch.int32, device=dev)
    nbytes = lib.sa_nsa_workspace_size(B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk)
    ws = _workspace(nbytes, dev)
    with torch.cuda.device(dev):
        check(lib.sa_nsa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(gates), B, T, Hq, Hkv, d, cmp_len,
                             cmp_stride, sel_block, sel_topk, window, float(scale), _ptr(out),
                             _ptr(lse3), _ptr(sel), _ptr(ws), nbytes, _stream(dev)), "sa_nsa_fwd")
    return out, lse3, sel


def nsa_fwd_train(q, k, v, gates, cmp_len: int, cmp_stride: int, sel_block: int, sel_topk: int,
                  window: int, scale: Optional[float] = None):
    """NSA forward that also returns what the backward needs (sa_nsa_fwd_train).

    Returns (out bf16 [B,T,Hq,d], lse_branches fp32 [B,T,Hq,3],
    sel_idx int32 [B,T,Hkv,sel_topk], o_branches fp32 [3,B,T,Hq,d]).
    """
    lib = _lib.load()
    dev = q.device
    _need(q, "q", torch.bfloat16, dev, 4)
    _need(k, "k", torch.bfloat16, dev, 4)
    _need(v, "v", torch.bfloat16, dev, 4)
    _need(gates, "gates", torch.float32, dev, 4)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, d) or v.shape != k.shape or gates.shape != (B, T, Hq, 3):
        raise ValueError("nsa_fwd_train: shape mismatch")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device=dev)
    lse3 = torch.empty((B, T, Hq, 3), dtype=torch.float32, device=dev)
    sel = torch.empty((B, T, Hkv, sel_topk), dtype=torch.int32, device=dev)
    o3 = torch.empty((3, B, T, Hq, d), dtype=torch.float32, device=dev)
    nbytes = lib.sa_nsa_workspace_size(B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk)
    ws = _workspace(nbytes, dev)
    with torch.cuda.device(dev):
        check(lib.sa_nsa_fwd_train(_ptr(q), _ptr(k), _ptr(v), _ptr(gates), B, T, Hq, Hkv, d, cmp_len,
                                   cmp_stride, sel_block, sel_topk, window, float(scale), _ptr(out),
                                   _ptr(lse3), _ptr(sel), _ptr(o3), _ptr(ws), nbytes, _stream(dev)),
              "sa_nsa_fwd_train")
    return out, lse3, sel, o3


def nsa_bwd(q, k, v, gates, dout, o_branches, lse_branches, sel_idx, cmp_len: int, cmp_stride: int,
            sel_block: int, sel_topk: int, window: int, scale: Optional[float] = None):
    """NSA backward (sa_nsa_bwd) with the forward's block choice held fixed.

    o_branches, lse_branches and sel_idx are nsa_fwd_train's.  Returns
    (dq fp32 [B,T,Hq,d], dk fp32 [B,T,Hkv,d], dv fp32 [B,T,Hkv,d],
    dgates fp32 [B,T,Hq,3]).
    """
    lib = _lib.load()
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _need(t, n, torch.bfloat16, dev, 4)
    _need(gates, "gates", torch.float32, dev, 4)
    _need(o_branches, "o_branches", torch.float32, dev, 5)
    _need(lse_branches, "lse_branches", torch.float32, dev, 4)
    _need(sel_idx, "sel_idx", torch.int32, dev, 4)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if (k.shape != (B, T, Hkv, d) or v.shape != k.shape or dout.shape != q.shape
            or gates.shape != (B, T, Hq, 3) or o_branches.shape != (3, B, T, Hq, d)
            or lse_branches.shape != (B, T, Hq, 3) or sel_idx.shape != (B, T, Hkv, sel_topk)):
        raise ValueError("nsa_bwd: shape mismatch")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty((B, T, Hq, d), dtype=torch.float32, device=dev)
    dk = torch.empty((B, T, Hkv, d), dtype=torch.float32, device=dev)
    dv = torch.empty((B, T, Hkv, d), dtype=torch.float32, device=dev)
    dg = torch.empty((B, T, Hq, 3), dtype=torch.float32, device=dev)
    nbytes = lib.sa_nsa_bwd_workspace_size(B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk)
    ws = _workspace(nbytes, dev)
    with torch.cuda.device(dev):
        check(lib.sa_nsa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(dout), _ptr(o_branches),
                             _ptr(lse_branches), _ptr(sel_idx), B, T, Hq, Hkv, d, cmp_len, cmp_stride,
                             sel_block, sel_topk, window, float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(dg), _ptr(ws), nbytes, _stream(dev)), "sa_nsa_bwd")
    return dq, dk, dv, dg


def full_attn_topk(q, k, v, topk: int, window: int, scale: Optional[float] = None,
                   out=None, lse=None, out_idx=None, workspace=None):
    """A full-attention layer as an exact indexer (sa_full_attn_topk).

    q bf16 [B,T,Hq,d], k/v bf16 [B,T,Hkv,d].  Returns (out bf16 [B,T,Hq,d],
    lse fp32 [B,T,Hq], idx int32 [B,T,topk+window]): the full layer's causal
    attention and, for the sparse layers, the forced window plus the top-k
    keys by the full layer's head-summed attention probabilities.
    """
    lib = _lib.load()
    dev = q.device
    _need(q, "q", torch.bfloat16, dev, 4)
    _need(k, "k", torch.bfloat16, dev, 4)
    _need(v, "v", torch.bfloat16, dev, 4)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, d) or v.shape != k.shape:
        raise ValueError("full_attn_topk: shape mismatch")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, T, Hq), dtype=torch.float32, device=dev)
    if out_idx is None:
        out_idx = torch.empty((B, T, topk + window), dtype=torch.int32, device=dev)
    nbytes = lib.sa_full_attn_topk_workspace_size(B, T, Hq, Hkv, d, topk, window)
    ws = workspace if workspace is not None else _workspace(nbytes, dev)
    with torch.cuda.device(dev):
        check(lib.sa_full_attn_topk(_ptr(q), _ptr(k), _ptr(v), B, T, Hq, Hkv, d, float(scale), topk,
                                    window, _ptr(out), _ptr(lse), _ptr(out_idx), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(dev)), "sa_full_attn_topk")
    return out, lse, out_idx


# --------------------------------------------------------------- IndexCache --
def dsa_decode_layers(pattern: str, layers, topk: int, window: int = 0, n_split: int = 1,
                      q_pos0: Optional[int] = None, scale: Optional[float] = None,
                      outs=None, lses=None, idx_cache=None, workspace=None):
    """IndexCache layer loop (sa_dsa_decode_layers).

    layers: list of dicts with q, k, v, q_idx, k_idx, w (same shapes for every
    layer).  F layers run the indexer, S layers reuse the cached indices.
    Returns (outs, lses, idx_cache).
    """
    lib = _lib.load()
    n = len(layers)
    if len(pattern) < n:
        raise ValueError("pattern shorter than the layer list")
    l0 = layers[0]
    dev = l0["q"].device
    B, Tq, Hq, d = l0["q"].shape
    L, Hkv = l0["k"].shape[1], l0["k"].shape[2]
    Hi, di = l0["q_idx"].shape[2], l0["q_idx"].shape[3]
    for ly in layers:
        _need(ly["q"], "q", torch.bfloat16, dev, 4)
        _need(ly["k"], "k", torch.bfloat16, dev, 4)
        _need(ly["v"], "v", torch.bfloat16, dev, 4)
        _need(ly["q_idx"], "q_idx", torch.int8, dev, 4)
        _need(ly["k_idx"], "k_idx", torch.int8, dev, 3)
        _need(ly["w"], "w", torch.int32, dev, 3)
    pos0 = L - Tq if q_pos0 is None else int(q_pos0)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if outs is None:
        outs = [torch.empty((B, Tq, Hq, d), dtype=torch.bfloat16, device=dev) for _ in range(n)]
    if lses is None:
        lses = [torch.empty((B, Tq, Hq), dtype=torch.float32, device=dev) for _ in range(n)]
    if idx_cache is None:
        idx_cache = torch.empty((B, Tq, topk + window), dtype=torch.int32, device=dev)
    arr = (sa_dsa_layer * n)()
    for i, ly in enumerate(layers):
        arr[i] = sa_dsa_layer(ly["q"].data_ptr(), ly["k"].data_ptr(), ly["v"].data_ptr(),
                              ly["q_idx"].data_ptr(), ly["k_idx"].data_ptr(), ly["w"].data_ptr(),
                              outs[i].data_ptr(), lses[i].data_ptr())
    nbytes = lib.sa_dsa_decode_layers_workspace_size(B, Tq, L, Hq, d, Hi, di, topk, window, n_split)
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, dev)
    with torch.cuda.device(dev):
        check(lib.sa_dsa_decode_layers(pattern.encode(), n, arr, B, Tq, L, Hq, Hkv, d, Hi, di,
                                       pos0, topk, window, float(scale), int(n_split),
                                       _ptr(idx_cache), _ptr(workspace), nbytes, _stream(dev)),
              "sa_dsa_decode_layers")
    return outs, lses, idx_cache


def dsa_decode_workspace_bytes(B, Tq, L, Hq, d, Hi, di, topk, window=0, n_split=1) -> int:
    return int(_lib.load().sa_dsa_decode_layers_workspace_size(B, Tq, L, Hq, d, Hi, di, topk,
                                                               window, n_split))
