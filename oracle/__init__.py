"""CPU oracle for causal sparse attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  It wraps ``oracle.c`` (plain loops, int64 scores, fp64
attention, full-sort top-k; compiled with gcc + OpenMP into ``liboracle.so``)
and shares no code with the CUDA library.

Every function takes CPU torch tensors (bf16 / int8 / int32 / fp32, as the
input generators produce them) and returns numpy arrays.  ``rows`` selects a
subset of flat query rows (b * T + t); ``None`` means all rows.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
something other than itself (torch float64 scaled_dot_product_attention,
numpy einsum / lexsort, brute force on tiny inputs, closed forms and
invariants).  Two readings are this build's own (the NSA page gives no
formula for either): the NSA block-importance mapping and the NSA
candidate-block rule.  They are pinned to that reading by the hand-derived
table ``tests/golden/nsa_importance.txt`` (a case where mapping compressed
tokens by their end position, or taking b*sel_block < t, gives other
values), not to a published formula.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (-O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c11", "-shared",
                               "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int64
            D = ctypes.c_double
            lib.oracle_indexer_scores.argtypes = [P, P, P, I, I, I, I, I, I, P, I, P]
            lib.oracle_indexer_topk.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, I, P, P]
            lib.oracle_fixed_graph_row.argtypes = [I, I, ctypes.c_int, P, I]
            lib.oracle_fixed_graph_row.restype = ctypes.c_int64
            lib.oracle_sparse_attn.argtypes = [P, P, P, I, I, I, I, I, I, I, P, I, I,
                                               P, P, P, D, P, I, P, P, P, P]
            lib.oracle_lse_combine.argtypes = [P, P, I, I, I, P, P]
            lib.oracle_sparse_attn_bwd.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, I, I, D, P, P, P]
            lib.oracle_nsa_compress.argtypes = [P, P, I, I, I, I, I, I, P, P]
            lib.oracle_full_attn_topk.argtypes = [P, P, P, I, I, I, I, I, D, I, I, P, I, P, P, P, P]
            lib.oracle_nsa_bwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, D,
                                           P, P, P, P]
            lib.oracle_nsa_fwd.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, I, D,
                                           P, I, P, P, P, P, P, P]
            for name in ("oracle_indexer_scores", "oracle_indexer_topk",
                         "oracle_sparse_attn", "oracle_sparse_attn_bwd", "oracle_lse_combine",
                         "oracle_nsa_compress", "oracle_nsa_fwd", "oracle_nsa_bwd",
                         "oracle_full_attn_topk"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc == 1:
        raise OracleError(f"{what}: invalid argument")
    if rc == 2:
        raise OracleError(f"{what}: index out of range or in the future")
    if rc != 0:
        raise OracleError(f"{what}: status {rc}")


def _np(t, dtype):
    """torch CPU tensor (or numpy array) -> contiguous numpy array of dtype."""
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        t = t.numpy()
    return np.ascontiguousarray(t, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows, n_all):
    if rows is None:
        return None, n_all
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    return r, int(r.size)


# --------------------------------------------------------------------------
def indexer_scores(q_idx, k_idx, w, q_pos0=0, rows=None):
    """Exact int64 indexer scores I(t, j) (IndexCache page, body).

    q_idx [B,Tq,Hi,di] int8, k_idx [B,L,di] int8, w [B,Tq,Hi] int32.
    Returns [n_rows, L] int64 with INT64_MIN after the query position.
    """
    lib = _load()
    B, Tq, Hi, di = q_idx.shape
    L = k_idx.shape[1]
    q = _np(q_idx, np.int8); k = _np(k_idx, np.int8); ww = _np(w, np.int32)
    r, n = _rows(rows, B * Tq)
    out = np.empty((n, L), dtype=np.int64)
    _check(lib.oracle_indexer_scores(_ptr(q), _ptr(k), _ptr(ww), B, Tq, L, Hi, di,
                                     q_pos0, _ptr(r), n, _ptr(out)), "indexer_scores")
    return out


def indexer_topk(q_idx, k_idx, w, topk, window=0, q_pos0=0, rows=None):
    """Causal top-k with a forced window (IndexCache page; HySparse2 page).

    Returns (idx [n_rows, topk+window] int32 ascending, -1 padded,
    count [n_rows] int32).
    """
    lib = _load()
    B, Tq, Hi, di = q_idx.shape
    L = k_idx.shape[1]
    q = _np(q_idx, np.int8); k = _np(k_idx, np.int8); ww = _np(w, np.int32)
    r, n = _rows(rows, B * Tq)
    K = topk + window
    idx = np.empty((n, K), dtype=np.int32)
    cnt = np.empty((n,), dtype=np.int32)
    _check(lib.oracle_indexer_topk(_ptr(q), _ptr(k), _ptr(ww), B, Tq, L, Hi, di, q_pos0,
                                   topk, window, _ptr(r), n, _ptr(idx), _ptr(cnt)),
           "indexer_topk")
    return idx, cnt


def fixed_graph(T, window, dilated=True, q_pos0=0, Tq=None, cap=None):
    """Fixed index sets of the SpatialLM page for positions q_pos0 .. q_pos0+Tq-1.

    Returns (idx [Tq, cap] int32 ascending, -1 padded, count [Tq]).
    """
    lib = _load()
    Tq = T if Tq is None else Tq
    if cap is None:
        cap = window + (64 if dilated else 0)
    idx = np.empty((Tq, cap), dtype=np.int32)
    cnt = np.empty((Tq,), dtype=np.int32)
    for t in range(Tq):
        n = lib.oracle_fixed_graph_row(q_pos0 + t, window, 1 if dilated else 0,
                                       idx[t].ctypes.data_as(ctypes.c_void_p), cap)
        if n < 0:
            raise OracleError("fixed_graph: cap too small")
        cnt[t] = n
    return idx, cnt


def sparse_attn(q, k, v, idx, scale=None, q_pos0=0, cq=None, ck=None, beta=None,
                rows=None, want_stats=False):
    """fp64 attention over explicit index lists.

    q [B,Tq,Hq,d], k/v [B,L,Hkv,d] bf16; idx [B,Tq,K] or [B,Tq,idx_heads,K]
    int32 (-1 padded).  Returns (out [n_rows,Hq,d] fp64, lse [n_rows,Hq]) and,
    with want_stats, also (psum [n_rows,Hq], maxj [n_rows]).
    """
    lib = _load()
    B, Tq, Hq, d = q.shape
    L, Hkv = k.shape[1], k.shape[2]
    ii = _np(idx, np.int32)
    if ii.ndim == 3:
        ii = ii.reshape(B, Tq, 1, ii.shape[-1])
    idx_heads, K = ii.shape[2], ii.shape[3]
    qq, kk, vv = _np(q, np.uint16), _np(k, np.uint16), _np(v, np.uint16)
    cqa = None if cq is None else _np(cq, np.float32)
    cka = None if ck is None else _np(ck, np.float32)
    ba = None if beta is None else _np(beta, np.float32)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r, n = _rows(rows, B * Tq)
    out = np.empty((n, Hq, d), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    psum = np.empty((n, Hq), dtype=np.float64)
    maxj = np.empty((n,), dtype=np.int64)
    _check(lib.oracle_sparse_attn(_ptr(qq), _ptr(kk), _ptr(vv), B, Tq, L, Hq, Hkv, d, q_pos0,
                                  _ptr(ii), idx_heads, K, _ptr(cqa), _ptr(cka), _ptr(ba),
                                  float(scale), _ptr(r), n, _ptr(out), _ptr(lse),
                                  _ptr(psum), _ptr(maxj)), "sparse_attn")
    if want_stats:
        return out, lse, psum, maxj
    return out, lse


def sparse_attn_bwd(q, k, v, dout, idx, scale=None, q_pos0=0):
    """fp64 backward of attention over explicit index lists (no bias).

    q/dout [B,Tq,Hq,d] bf16, k/v [B,L,Hkv,d] bf16, idx [B,Tq,K] or
    [B,Tq,idx_heads,K] int32 (-1 padded).  Returns (dq [B,Tq,Hq,d],
    dk [B,L,Hkv,d], dv [B,L,Hkv,d]) in fp64.
    """
    lib = _load()
    B, Tq, Hq, d = q.shape
    L, Hkv = k.shape[1], k.shape[2]
    ii = _np(idx, np.int32)
    if ii.ndim == 3:
        ii = ii.reshape(B, Tq, 1, ii.shape[-1])
    idx_heads, K = ii.shape[2], ii.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq = np.empty((B, Tq, Hq, d), dtype=np.float64)
    dk = np.empty((B, L, Hkv, d), dtype=np.float64)
    dv = np.empty((B, L, Hkv, d), dtype=np.float64)
    _check(lib.oracle_sparse_attn_bwd(_ptr(_np(q, np.uint16)), _ptr(_np(k, np.uint16)),
                                      _ptr(_np(v, np.uint16)), _ptr(_np(dout, np.uint16)),
                                      B, Tq, L, Hq, Hkv, d, q_pos0, _ptr(ii), idx_heads, K,
                                      float(scale), _ptr(dq), _ptr(dk), _ptr(dv)),
           "sparse_attn_bwd")
    return dq, dk, dv


def lse_combine(part_o, part_lse):
    """Distributed-softmax merge (Star Attention page).

    part_o [S, rows, d], part_lse [S, rows] (any float type) ->
    (out [rows, d], lse [rows]) in fp64.
    """
    lib = _load()
    po = _np(part_o, np.float64)
    pl = _np(part_lse, np.float64)
    S, R, d = po.shape
    out = np.empty((R, d), dtype=np.float64)
    lse = np.empty((R,), dtype=np.float64)
    _check(lib.oracle_lse_combine(_ptr(po), _ptr(pl), S, R, d, _ptr(out), _ptr(lse)),
           "lse_combine")
    return out, lse


def nsa_compress(k, v, cmp_len, cmp_stride):
    """NSA coarse compression: mean of each length-cmp_len window (fp64)."""
    lib = _load()
    B, T, Hkv, d = k.shape
    nc = (T - cmp_len) // cmp_stride + 1 if T >= cmp_len else 0
    kc = np.empty((B, nc, Hkv, d), dtype=np.float64)
    vc = np.empty((B, nc, Hkv, d), dtype=np.float64)
    if nc:
        _check(lib.oracle_nsa_compress(_ptr(_np(k, np.uint16)), _ptr(_np(v, np.uint16)),
                                       B, T, Hkv, d, cmp_len, cmp_stride, _ptr(kc), _ptr(vc)),
               "nsa_compress")
    return kc, vc


def nsa_fwd(q, k, v, gates, cmp_len, cmp_stride, sel_block, sel_topk, window,
            scale=None, rows=None, sel_override=None):
    """NSA forward (Native Sparse Attention page) in fp64.

    Returns dict: out [n,Hq,d], o_branch [3,n,Hq,d], lse_branch [n,Hq,3],
    sel_idx [n,Hkv,sel_topk], imp [n,Hkv,n_blocks].

    The importance mapping (selection block b sums the compressed-branch
    probabilities of compressed tokens whose start lies in
    [b*sel_block, (b+1)*sel_block), over the heads of the KV group) and the
    candidate rule (blocks with b*sel_block <= t, none forced) are readings of
    a page that gives no formula.  They are pinned to that reading by a
    hand-derived table (tests/golden/nsa_importance.txt), not to a published
    formula.
    """
    lib = _load()
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r, n = _rows(rows, B * T)
    nb = (T + sel_block - 1) // sel_block
    so = None if sel_override is None else _np(sel_override, np.int32)
    out = np.empty((n, Hq, d), dtype=np.float64)
    ob = np.empty((3, n, Hq, d), dtype=np.float64)
    lb = np.empty((n, Hq, 3), dtype=np.float64)
    si = np.empty((n, Hkv, sel_topk), dtype=np.int32)
    imp = np.empty((n, Hkv, nb), dtype=np.float64)
    _check(lib.oracle_nsa_fwd(_ptr(_np(q, np.uint16)), _ptr(_np(k, np.uint16)),
                              _ptr(_np(v, np.uint16)), _ptr(_np(gates, np.float32)),
                              B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk,
                              window, float(scale), _ptr(r), n, _ptr(so), _ptr(out),
                              _ptr(ob), _ptr(lb), _ptr(si), _ptr(imp)), "nsa_fwd")
    return {"out": out, "o_branch": ob, "lse_branch": lb, "sel_idx": si, "imp": imp}


def nsa_bwd(q, k, v, gates, dout, sel_idx, cmp_len, cmp_stride, sel_block, sel_topk,
            window, scale=None):
    """fp64 NSA backward (Native Sparse Attention page) with the block choice
    sel_idx [B*T, Hkv, sel_topk] (the forward's) held fixed.

    Returns dict: dq [B,T,Hq,d], dk / dv [B,T,Hkv,d], dgates [B,T,Hq,3]
    (gradient with respect to the post-sigmoid gate values).
    """
    lib = _load()
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    si = _np(sel_idx, np.int32).reshape(B * T, Hkv, sel_topk)
    dq = np.empty((B, T, Hq, d), dtype=np.float64)
    dk = np.empty((B, T, Hkv, d), dtype=np.float64)
    dv = np.empty((B, T, Hkv, d), dtype=np.float64)
    dg = np.empty((B, T, Hq, 3), dtype=np.float64)
    _check(lib.oracle_nsa_bwd(_ptr(_np(q, np.uint16)), _ptr(_np(k, np.uint16)),
                              _ptr(_np(v, np.uint16)), _ptr(_np(gates, np.float32)),
                              _ptr(_np(dout, np.uint16)), _ptr(si), B, T, Hq, Hkv, d,
                              cmp_len, cmp_stride, sel_block, sel_topk, window, float(scale),
                              _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg)), "nsa_bwd")
    return {"dq": dq, "dk": dk, "dv": dv, "dgates": dg}


def full_attn_topk(q, k, v, topk, window, scale=None, rows=None, want_scores=False):
    """A full-attention layer as an exact indexer (HySparse2 page), fp64.

    q [B,T,Hq,d], k/v [B,T,Hkv,d] bf16.  Returns (out [n,Hq,d], lse [n,Hq],
    idx [n, topk+window] int32) and, with want_scores, scores [n, T]: the
    full layer's attention probability on each key summed over all heads.
    The set is the forced window plus the top-k of the other keys by
    (score desc, index asc), ascending and -1 padded.
    """
    lib = _load()
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r, n = _rows(rows, B * T)
    out = np.empty((n, Hq, d), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    idx = np.empty((n, topk + window), dtype=np.int32)
    sc = np.empty((n, T), dtype=np.float64) if want_scores else None
    _check(lib.oracle_full_attn_topk(_ptr(_np(q, np.uint16)), _ptr(_np(k, np.uint16)),
                                     _ptr(_np(v, np.uint16)), B, T, Hq, Hkv, d, float(scale),
                                     topk, window, _ptr(r), n, _ptr(out), _ptr(lse), _ptr(idx),
                                     _ptr(sc)), "full_attn_topk")
    if want_scores:
        return out, lse, idx, sc
    return out, lse, idx


def dsa_layers(pattern, layers, topk, window=0, q_pos0=None, scale=None):
    """IndexCache layer loop (IndexCache page, body).

    pattern: string of 'F'/'S', first char 'F'.  layers: list of dicts with
    q, k, v, q_idx, k_idx, w (one query token per sequence or a prefill).
    F layers run the indexer and replace the cached index buffer; S layers
    reuse the buffer of the nearest preceding F layer.
    Returns list of (idx, out, lse) per layer.
    """
    if not pattern or pattern[0] != "F" or any(c not in "FS" for c in pattern):
        raise OracleError("pattern must start with F and contain only F/S")
    res = []
    cached = None
    for ch, lay in zip(pattern, layers):
        B, Tq = lay["q"].shape[:2]
        L = lay["k"].shape[1]
        pos0 = (L - Tq) if q_pos0 is None else q_pos0
        if ch == "F":
            idx, _ = indexer_topk(lay["q_idx"], lay["k_idx"], lay["w"], topk, window, pos0)
            cached = idx.reshape(B, Tq, -1)
        out, lse = sparse_attn(lay["q"], lay["k"], lay["v"], cached, scale=scale, q_pos0=pos0)
        res.append((cached.copy(), out, lse))
    return res
