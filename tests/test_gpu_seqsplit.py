"""GPU check of the sequence-split decode (fixed_pattern_sparse_sa_b200.seqsplit):
the keys of each sequence split by position over R ranks, emulated in one
process on one GPU (each rank's phases run in turn, the exchanges are
stacks; no kernel waits on another rank's).  The merged selection must equal
the single-GPU selection bit for bit, and the merged attention must match
the oracle over the whole sequence."""
import numpy as np
import pytest
import torch

import oracle
from fixed_pattern_sparse_sa_b200 import api, inputs, seqsplit
from _parity import assert_lse_close, assert_out_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("window", [0, 64])
@pytest.mark.parametrize("bounds", [[0, 5000, 10000, 15000, 20000], [0, 3000, 11000, 20000]])
def test_seqsplit_decode_matches_single_gpu(cuda_ok, window, bounds):
    nseq, L, topk = 3, bounds[-1], 2048
    lay = to_dev(inputs.gen_decode_layer(nseq, L, 16, 1, 128, 8, 64, layer=0, seed=41))
    shards = [seqsplit.Shard(q=lay["q"], k=lay["k"][:, lo:hi].contiguous(), v=lay["v"][:, lo:hi].contiguous(),
                             q_idx=lay["q_idx"], k_idx=lay["k_idx"][:, lo:hi].contiguous(), w=lay["w"], key_lo=lo)
              for lo, hi in zip(bounds[:-1], bounds[1:])]
    out, lse, sel = seqsplit.emulated_step(shards, topk, window, L)
    api.check_device_status()
    one, _ = api.indexer_topk(lay["q_idx"], lay["k_idx"], lay["w"], topk, window, q_pos0=L - 1)
    np.testing.assert_array_equal(sel.cpu().numpy(), one.cpu().numpy())
    host = {k: v.cpu() for k, v in lay.items()}
    ref_idx, _ = oracle.indexer_topk(host["q_idx"], host["k_idx"], host["w"], topk, window, q_pos0=L - 1)
    np.testing.assert_array_equal(sel.cpu().numpy().reshape(ref_idx.shape), ref_idx)
    ro, rl = oracle.sparse_attn(host["q"], host["k"], host["v"], ref_idx.reshape(nseq, 1, -1), q_pos0=L - 1)
    assert_out_close(out, ro, "seqsplit out")
    assert_lse_close(lse, rl, "seqsplit lse")


def test_topk_merge_ties_and_window(cuda_ok):
    # heavy ties across parts: equal scores go to the lowest positions; window
    # positions are never ranked, they are appended
    rows, R, kc, topk, window, q_pos = 2, 3, 6, 5, 3, 40
    score = torch.tensor([[[7, 7, 7, 1, 9, -1]] * rows] * R, dtype=torch.int32)
    idx = torch.tensor([[[0, 1, 2, 3, 4, -1]] * rows] * R, dtype=torch.int32)
    offs = [0, 10, 36]                                   # part 2 holds positions 36..41 (38.. in the window)
    got, cnt = api.topk_merge(score.cuda(), idx.cuda(), offs, topk, window, q_pos)
    # ranked candidates (positions < 38): score 9 at 4 and 14; 7 at 0, 1, 2,
    # 10, 11, 12, 36, 37; 1 at 3 and 13.  Top 5: 4, 14 and the three lowest
    # 7s (0, 1, 2); then the window 38, 39, 40
    expect = [0, 1, 2, 4, 14, 38, 39, 40]
    assert got.cpu().tolist() == [expect] * rows
    assert cnt.cpu().tolist() == [8] * rows
