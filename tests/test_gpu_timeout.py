"""GPU check of the timeout path: a kernel whose bounded wait runs out stops
cleanly, reports SA_ERR_TIMEOUT through sa_check_device_status, and leaves
the context usable.  The wait is made to run out without any fault: the
library's stall hook stops the NSA tensor-core branch kernels from issuing
their loads, so their first barrier wait is on a barrier that nothing will
complete, and the spin limit is set to a few milliseconds.  No TMA or MMA is
in flight when the kernel gives up."""
import numpy as np
import pytest

import oracle
from fixed_pattern_sparse_sa_b200 import _lib, api, inputs
from fixed_pattern_sparse_sa_b200._lib import SAError
from _parity import assert_lse_close, assert_out_close, to_dev

pytestmark = pytest.mark.gpu

CFG = dict(cmp_len=32, cmp_stride=16, sel_block=64, sel_topk=8, window=128)


def test_stalled_wait_reports_timeout_then_recovers(cuda_ok):
    g = inputs.gen_nsa(1, 333, 32, 2, 128, seed=77)
    gd = to_dev(g)
    api.check_device_status()                       # start from a clean error word
    try:
        api.debug_set_spin_limit(20_000_000)          # ~10 ms at 1.9 GHz
        api.debug_inject_stall(True)
        api.nsa_fwd(gd["q"], gd["k"], gd["v"], gd["gates"], **CFG)
        with pytest.raises(SAError) as ei:
            api.check_device_status()
        assert ei.value.status == _lib.SA_ERR_TIMEOUT, str(ei.value)
        assert "spin limit" in str(ei.value)
    finally:
        api.debug_inject_stall(False)
        api.debug_set_spin_limit(0)
    # the error word was cleared by the check, and the next call is correct
    out, lse3, sel = api.nsa_fwd(gd["q"], gd["k"], gd["v"], gd["gates"], **CFG)
    api.check_device_status()
    rows = np.arange(333)
    ref = oracle.nsa_fwd(g["q"], g["k"], g["v"], g["gates"], rows=rows, **CFG)
    # compared on the rows whose block choice equals the oracle's (near ties
    # in the float importances may pick another block of equal weight)
    same = np.all(np.sort(sel.cpu().numpy().reshape(333, -1), axis=1)
                  == np.sort(ref["sel_idx"].reshape(333, -1), axis=1), axis=1)
    keep = np.nonzero(same)[0]
    assert len(keep) >= 333 - 3
    assert_out_close(out.reshape(-1, 32, 128)[keep], ref["out"][keep], "nsa out after timeout")
    assert_lse_close(lse3.reshape(-1, 32, 3)[keep], ref["lse_branch"][keep], "nsa lse after timeout")


def test_stalled_exact_indexer_reports_timeout_then_recovers(cuda_ok):
    """The exact indexer's tensor-core kernels (the full layer and the score
    pass) under the stall hook: nothing is loaded or multiplied, their waits
    run out and the call reports SA_ERR_TIMEOUT.  The workspace and the LSE
    are zero-filled first, so the select that follows reads valid (zero)
    scores.  The next call matches the oracle."""
    import torch
    from test_gpu_full_indexer import _check_out, _check_sets
    B, T, Hq, Hkv, d, topk, window = 1, 300, 16, 1, 128, 64, 16
    g = inputs.gen_dsa(B, T, Hq, Hkv, d, 1, 32, seed=T + d)
    q, k, v = (g[n].cuda() for n in ("q", "k", "v"))
    lib = _lib.load()
    ws = torch.zeros(lib.sa_full_attn_topk_workspace_size(B, T, Hq, Hkv, d, topk, window),
                     dtype=torch.uint8, device="cuda")
    out = torch.zeros((B, T, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, T, Hq), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, T, topk + window), dtype=torch.int32, device="cuda")
    api.check_device_status()
    try:
        api.debug_set_spin_limit(20_000_000)
        api.debug_inject_stall(True)
        api.full_attn_topk(q, k, v, topk, window, out=out, lse=lse, out_idx=idx, workspace=ws)
        with pytest.raises(SAError) as ei:
            api.check_device_status()
        assert ei.value.status == _lib.SA_ERR_TIMEOUT, str(ei.value)
    finally:
        api.debug_inject_stall(False)
        api.debug_set_spin_limit(0)
    out, lse, idx = api.full_attn_topk(q, k, v, topk, window)
    api.check_device_status()
    ref_out, ref_lse, ref_idx, sc = oracle.full_attn_topk(g["q"], g["k"], g["v"], topk, window,
                                                          want_scores=True)
    _check_out(out, lse, ref_out, ref_lse)
    _check_sets(idx, ref_idx, sc, topk, window, T, None)
