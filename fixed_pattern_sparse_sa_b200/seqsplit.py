"""Decode over a sequence whose keys are split by position across GPUs.

Star Attention page ("NVIDIA AI Research presenta Star Attention ...",
body): the context is spread over hosts and their results are merged by a
distributed softmax, with little data crossing between them.  Here each rank
holds the K, V and indexer keys of positions [key_lo, key_lo + S) of every
sequence; the decode query of a sequence (at the last position, L_total - 1)
is on every rank.  One step:

  phase 1 (per rank)   exact top-(topk + window) of the rank's own keys, and
                       their indexer scores;
  exchange             all-gather of the (score, index) candidates;
  phase 2 (per rank)   exact global top-k of the candidates with the forced
                       window (the same selection as on one GPU), the rank's
                       share of it, and the rank's partial attention
                       (fp32 out and lse of two split pieces);
  exchange             all-gather of the partial results;
  phase 3              log-sum-exp merge into out / lse.

Only the library's kernels compute; this module moves tensors between the
phases.  `exchange(t)` stacks one tensor per rank along a new first axis:
torch.distributed.all_gather_into_tensor on a process group, or a plain
stack when the ranks are emulated in one process.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Sequence

import torch

from . import api


@dataclass
class Shard:
    q: torch.Tensor        # bf16 [B, 1, Hq, d]   the decode queries
    k: torch.Tensor        # bf16 [B, S, Hkv, d]  this rank's keys
    v: torch.Tensor        # bf16 [B, S, Hkv, d]
    q_idx: torch.Tensor    # int8 [B, 1, Hi, di]
    k_idx: torch.Tensor    # int8 [B, S, di]
    w: torch.Tensor        # int32 [B, 1, Hi]
    key_lo: int            # position of this rank's first key


def phase1(sh: Shard, topk: int, window: int, ops=api):
    """Local candidates: the exact top-(topk + window) of this rank's keys
    (every local key precedes the decode query) and their scores."""
    S = sh.k.shape[1]
    kc = topk + window
    idx, _ = ops.indexer_topk(sh.q_idx, sh.k_idx, sh.w, kc, 0, q_pos0=S - 1)
    score = ops.indexer_scores_at(sh.q_idx, sh.k_idx, sh.w, idx)
    return score, idx


def phase2(sh: Shard, cand_score, cand_idx, key_los: Sequence[int], topk: int, window: int, L_total: int,
           ops=api):
    """Global selection from the gathered candidates [R, B, 1, kc], then the
    rank's partial attention over the selected keys it holds."""
    R, B = cand_score.shape[0], cand_score.shape[1]
    sel, _ = ops.topk_merge(cand_score.reshape(R, B, -1), cand_idx.reshape(R, B, -1), key_los, topk, window,
                            L_total - 1)
    S = sh.k.shape[1]
    local = ops.index_shard(sel, sh.key_lo, sh.key_lo + S).reshape(B, 1, -1)
    _, _, po, pl = ops.sparse_attn_fwd(sh.q, sh.k, sh.v, local, n_split=2, q_pos0=S - 1, return_partials=True)
    return sel.reshape(B, 1, -1), po, pl


def phase3(part_o, part_lse, ops=api):
    """Merge the gathered partial results [R, 2, B, 1, Hq, d] / [R, 2, B, 1, Hq]."""
    R, P = part_o.shape[0], part_o.shape[1]
    B, _, Hq, d = part_o.shape[2:]
    out, lse = ops.lse_combine(part_o.reshape(R * P, B * Hq, d), part_lse.reshape(R * P, B * Hq))
    return out.reshape(B, 1, Hq, d), lse.reshape(B, 1, Hq)


def decode_step(sh: Shard, topk: int, window: int, L_total: int,
                exchange: Callable[[torch.Tensor], torch.Tensor], key_los: Sequence[int], ops=api):
    """One decode step on this rank; every rank calls it with its own shard
    (the same collectives in the same order on every rank)."""
    score, idx = phase1(sh, topk, window, ops)
    cs, ci = exchange(score), exchange(idx)
    sel, po, pl = phase2(sh, cs, ci, key_los, topk, window, L_total, ops)
    out, lse = phase3(exchange(po), exchange(pl), ops)
    return out, lse, sel


def dist_exchange(group=None):
    """All-gather over a torch.distributed process group (NCCL between GPUs,
    gloo on CPU), stacked along a new first axis in rank order."""
    import torch.distributed as dist

    def ex(t: torch.Tensor) -> torch.Tensor:
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)
    return ex


def emulated_step(shards: Sequence[Shard], topk: int, window: int, L_total: int, ops=api):
    """All ranks' phases run in this process on one device, the exchanges as
    stacks: the same kernels and data flow as decode_step over R GPUs (no
    kernel of one rank waits on another's)."""
    key_los = [s.key_lo for s in shards]
    p1 = [phase1(s, topk, window, ops) for s in shards]
    cs = torch.stack([x[0] for x in p1])
    ci = torch.stack([x[1] for x in p1])
    p2 = [phase2(s, cs, ci, key_los, topk, window, L_total, ops) for s in shards]
    out, lse = phase3(torch.stack([x[1] for x in p2]), torch.stack([x[2] for x in p2]), ops)
    return out, lse, p2[0][0]
