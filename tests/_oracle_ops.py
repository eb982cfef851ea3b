"""CPU stand-ins (test infrastructure) for the library calls of the
sequence-split decode driver, built on the fp64 / int64 oracle, so that the
driver's data flow between ranks runs on CPU gloo ranks.  The merge step is
written here from its definition (exact top-k of the gathered candidates by
(score desc, position asc), the forced window appended) and checked against
the oracle's selection over the whole sequence by the tests."""
import numpy as np
import torch

import oracle


def indexer_topk(q_idx, k_idx, w, topk, window, q_pos0):
    idx, cnt = oracle.indexer_topk(q_idx, k_idx, w, topk, window, q_pos0=q_pos0)
    B, Tq = q_idx.shape[:2]
    return torch.from_numpy(idx).reshape(B, Tq, -1), torch.from_numpy(cnt).reshape(B, Tq)


def indexer_scores_at(q_idx, k_idx, w, idx):
    B, Tq = q_idx.shape[:2]
    sc = oracle.indexer_scores(q_idx, k_idx, w, q_pos0=k_idx.shape[1] - Tq)     # [B*Tq, L]
    ii = idx.reshape(B * Tq, -1).numpy()
    out = np.where(ii >= 0, np.take_along_axis(sc, np.maximum(ii, 0), axis=1), np.iinfo(np.int32).min)
    return torch.from_numpy(out.astype(np.int32)).reshape(idx.shape)


def topk_merge(cand_score, cand_idx, part_off, topk, window, q_pos):
    R, rows, kc = cand_score.shape
    wlo = q_pos - window + 1 if window > 0 else q_pos + 1
    wc = min(window, q_pos + 1) if window > 0 else 0
    out = np.full((rows, topk + window), -1, dtype=np.int32)
    cnt = np.zeros(rows, dtype=np.int32)
    for r in range(rows):
        cands = []
        for p in range(R):
            for e in range(kc):
                j = int(cand_idx[p, r, e])
                if j < 0:
                    continue
                gj = j + int(part_off[p])
                if gj < wlo:
                    cands.append((-int(cand_score[p, r, e]), gj))
        chosen = sorted(sorted(cands)[:topk], key=lambda x: x[1])
        row = [gj for _, gj in chosen] + list(range(q_pos - wc + 1, q_pos + 1))
        out[r, :len(row)] = row
        cnt[r] = len(row)
    return torch.from_numpy(out), torch.from_numpy(cnt)


def index_shard(idx, key_lo, key_hi):
    ii = idx.numpy()
    return torch.from_numpy(np.where((ii >= key_lo) & (ii < key_hi), ii - key_lo, -1).astype(np.int32))


def sparse_attn_fwd(q, k, v, idx, n_split, q_pos0, return_partials):
    """Partial results as two pieces: the whole list, and an empty piece."""
    B, Tq, Hq, d = q.shape
    o, l = oracle.sparse_attn(q, k, v, idx, q_pos0=q_pos0)
    po = torch.zeros((n_split, B, Tq, Hq, d), dtype=torch.float64)
    pl = torch.full((n_split, B, Tq, Hq), float("-inf"), dtype=torch.float64)
    po[0] = torch.from_numpy(o).reshape(B, Tq, Hq, d)
    pl[0] = torch.from_numpy(l).reshape(B, Tq, Hq)
    return None, None, po, pl


def lse_combine(part_o, part_lse):
    o, l = oracle.lse_combine(part_o, part_lse)
    return torch.from_numpy(o), torch.from_numpy(l)
