"""Seeded synthetic inputs for the five sparse-attention workloads.

This module only draws random tensors; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle take their inputs from it.
Every tensor comes from one ``torch.Generator`` seeded with ``seed`` and drawn
in the order written in each function, so a workload is reproducible on any
machine with the same torch version.

bf16 tensors are drawn as fp32 N(0, 1) and rounded to bf16 (round to nearest
even).  Indexer tensors are int8 uniform on [-8, 8]; indexer head weights are
int32 uniform on [0, 4].

Workloads (sizes as named):
  tiny_dsa        1 x 512 tokens, 4 query heads / 1 KV head, d=64; indexer
                  2 heads, d=32; top-64 plus a forced window of 32.
  spatial16k      1 x 16384 tokens, 8 heads (one KV head each), d=64; fixed
                  graph = self + 64 predecessors + offsets 2^i < t; 3-D fp32
                  coordinates N(0, 1), beta = 0.5 for every head.
  dsa_prefill64k  1 x 65536 tokens, 16 query heads / 1 KV head, d=128;
                  indexer 8 heads, d=64; top-2048.
  dsa_decode128k  32 sequences x 131072 cached tokens, one query token each,
                  16 query heads / 1 KV head, d=128, top-2048, 4 layers.
  nsa64k          1 x 65536 tokens, 64 query heads / 4 KV heads, d=128;
                  compression length 32 stride 16, top-16 of 64-token blocks,
                  window 512, sigmoid gates U(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

__all__ = [
    "WORKLOADS", "Workload", "gen_dsa", "gen_spatial", "gen_decode_layer",
    "gen_nsa",
]


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                    # "dsa", "spatial", "decode", "nsa"
    B: int
    T: int                       # query tokens (prefill) or cached tokens (decode)
    Hq: int
    Hkv: int
    d: int
    Hi: int = 0
    di: int = 0
    topk: int = 0
    window: int = 0
    layers: int = 1
    dilated: bool = False
    beta: float = 0.0
    cmp_len: int = 0
    cmp_stride: int = 0
    sel_block: int = 0
    sel_topk: int = 0
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny_dsa": Workload("tiny_dsa", "dsa", B=1, T=512, Hq=4, Hkv=1, d=64,
                         Hi=2, di=32, topk=64, window=32),
    # window counts the token itself: self + 64 predecessors = 65 positions
    "spatial16k": Workload("spatial16k", "spatial", B=1, T=16384, Hq=8, Hkv=8,
                           d=64, window=65, dilated=True, beta=0.5),
    "dsa_prefill64k": Workload("dsa_prefill64k", "dsa", B=1, T=65536, Hq=16,
                               Hkv=1, d=128, Hi=8, di=64, topk=2048, window=0),
    "dsa_decode128k": Workload("dsa_decode128k", "decode", B=32, T=131072,
                               Hq=16, Hkv=1, d=128, Hi=8, di=64, topk=2048,
                               window=0, layers=4),
    "nsa64k": Workload("nsa64k", "nsa", B=1, T=65536, Hq=64, Hkv=4, d=128,
                       cmp_len=32, cmp_stride=16, sel_block=64, sel_topk=16,
                       window=512),
}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn_bf16(shape, g, device="cpu"):
    return torch.randn(shape, generator=g, dtype=torch.float32,
                       device=device).to(torch.bfloat16)


def _randint(lo, hi_inclusive, shape, dtype, g, device="cpu"):
    return torch.randint(lo, hi_inclusive + 1, shape, generator=g,
                         dtype=torch.int64, device=device).to(dtype)


def gen_dsa(B, T, Hq, Hkv, d, Hi, di, seed=0, L=None):
    """DSA prefill inputs.  Draw order: q, k, v, q_idx, k_idx, w.

    q [B,T,Hq,d], k/v [B,L,Hkv,d] bf16; q_idx [B,T,Hi,di], k_idx [B,L,di] int8
    in [-8, 8]; w [B,T,Hi] int32 in [0, 4].  L defaults to T.
    """
    L = T if L is None else L
    g = _gen(seed)
    return {
        "q": _randn_bf16((B, T, Hq, d), g),
        "k": _randn_bf16((B, L, Hkv, d), g),
        "v": _randn_bf16((B, L, Hkv, d), g),
        "q_idx": _randint(-8, 8, (B, T, Hi, di), torch.int8, g),
        "k_idx": _randint(-8, 8, (B, L, di), torch.int8, g),
        "w": _randint(0, 4, (B, T, Hi), torch.int32, g),
    }


def gen_spatial(B, T, H, d, beta=0.5, seed=0, Hkv=None):
    """Fixed-graph inputs.  Draw order: q, k, v, cq, ck.

    q [B,T,H,d], k/v [B,T,Hkv,d] bf16; cq [B,T,H,3], ck [B,T,Hkv,3] fp32
    N(0, 1); beta [H] fp32 constant.
    """
    Hkv = H if Hkv is None else Hkv
    g = _gen(seed)
    return {
        "q": _randn_bf16((B, T, H, d), g),
        "k": _randn_bf16((B, T, Hkv, d), g),
        "v": _randn_bf16((B, T, Hkv, d), g),
        "cq": torch.randn((B, T, H, 3), generator=g, dtype=torch.float32),
        "ck": torch.randn((B, T, Hkv, 3), generator=g, dtype=torch.float32),
        "beta": torch.full((H,), float(beta), dtype=torch.float32),
    }


def gen_decode_layer(nseq, L, Hq, Hkv, d, Hi, di, layer, seed=0, device="cpu"):
    """One decode layer's inputs (each layer draws from seed + 1000*layer).

    Draw order: k cache, v cache, k_idx cache, q, q_idx, w.
    k/v [nseq,L,Hkv,d] bf16; k_idx [nseq,L,di] int8; q [nseq,1,Hq,d] bf16;
    q_idx [nseq,1,Hi,di] int8; w [nseq,1,Hi] int32.  The caches are large
    (1 GiB each at 32 x 131072 x 128), so callers may draw them directly on a
    CUDA device with that device's generator; the values then differ from a
    CPU draw but are just as reproducible.
    """
    g = _gen(seed + 1000 * layer, device)
    return {
        "k": _randn_bf16((nseq, L, Hkv, d), g, device),
        "v": _randn_bf16((nseq, L, Hkv, d), g, device),
        "k_idx": _randint(-8, 8, (nseq, L, di), torch.int8, g, device),
        "q": _randn_bf16((nseq, 1, Hq, d), g, device),
        "q_idx": _randint(-8, 8, (nseq, 1, Hi, di), torch.int8, g, device),
        "w": _randint(0, 4, (nseq, 1, Hi), torch.int32, g, device),
    }


def gen_nsa(B, T, Hq, Hkv, d, seed=0):
    """NSA inputs.  Draw order: q, k, v, gates.

    q [B,T,Hq,d], k/v [B,T,Hkv,d] bf16; gates [B,T,Hq,3] fp32 U(0, 1) (the
    branch gates are already sigmoid outputs).
    """
    g = _gen(seed)
    return {
        "q": _randn_bf16((B, T, Hq, d), g),
        "k": _randn_bf16((B, T, Hkv, d), g),
        "v": _randn_bf16((B, T, Hkv, d), g),
        "gates": torch.rand((B, T, Hq, 3), generator=g, dtype=torch.float32),
    }
