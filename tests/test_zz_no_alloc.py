"""GPU check of sa_sparse_attn_fwd_split_static, the split-KV attention entry
point that keeps its partial results in a fixed array inside the library
instead of allocating.  It is compared with sa_sparse_attn_fwd (caller-owned
partial buffers) on two calls in a row with different inputs, so a result
left over from the first call in the shared array would show up in the
second.  The file name sorts last so that it also runs after every other
GPU test in the same process.  The second call of a pair is also checked
against the CPU oracle directly, on the default gather kernel and, in a
fresh process, on the tcgen05 gather kernel (SA_ATTN_PATH=tc), which writes
its partials into the same array."""
import ctypes
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from fixed_pattern_sparse_sa_b200 import _lib, api
from fixed_pattern_sparse_sa_b200._lib import SAError
from _parity import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

SA_ERR_WORKSPACE = {v: k for k, v in _lib.STATUS.items()}["SA_ERR_WORKSPACE"]


def _case(B, T, Hq, Hkv, d, K, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(seed)
    idx = np.full((B, T, K), -1, dtype=np.int32)
    for b in range(B):
        for t in range(T):
            n = min(t + 1, K)
            idx[b, t, :n] = rng.choice(t + 1, size=n, replace=False)
    dev = torch.device("cuda:0")
    return (q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(idx).to(dev))


def _static_call(q, k, v, idx, n_split):
    """Direct C-ABI call; returns (status, out, lse)."""
    lib = _lib.load()
    B, Tq, Hq, d = q.shape
    L, Hkv = k.shape[1], k.shape[2]
    K = idx.shape[-1]
    out = torch.empty((B, Tq, Hq, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=q.device)
    st = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    rc = lib.sa_sparse_attn_fwd_split_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        B, Tq, L, Hq, Hkv, d, L - Tq, ctypes.c_void_p(idx.data_ptr()), 1, K,
        1.0 / math.sqrt(d), n_split, ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), st)
    return rc, out, lse


@pytest.mark.parametrize("d,n_split", [(128, 4), (64, 3)])
def test_static_split_matches_workspace_path_twice(cuda_ok, d, n_split):
    B, T, Hq, Hkv, K = 2, 96, 16, 2, 80
    for seed in (11, 12):
        q, k, v, idx = _case(B, T, Hq, Hkv, d, K, seed + d)
        rc, out, lse = _static_call(q, k, v, idx, n_split)
        assert rc == _lib.SA_OK, _lib.load().sa_last_error_string().decode()
        torch.cuda.synchronize()
        ref_out, ref_lse = api.sparse_attn_fwd(q, k, v, idx, n_split=n_split)
        torch.cuda.synchronize()
        assert_out_close(out, ref_out.double().cpu().numpy())
        assert_lse_close(lse, ref_lse.double().cpu().numpy())
    api.check_device_status()


def test_static_split_largest_fitting_case(cuda_ok):
    # n_split * rows * (d + 1) * 4 bytes: 4 * 2 * 128 * 16 * 129 * 4 = 8.45 MB
    # is too big; 3 splits (6.3 MB) fit.
    B, T, Hq, Hkv, d, K = 2, 128, 16, 2, 128, 200
    q, k, v, idx = _case(B, T, Hq, Hkv, d, K, 5)
    rc, _, _ = _static_call(q, k, v, idx, 4)
    assert rc == SA_ERR_WORKSPACE
    assert "built-in scratch" in _lib.load().sa_last_error_string().decode()
    rc, out, lse = _static_call(q, k, v, idx, 3)
    assert rc == _lib.SA_OK, _lib.load().sa_last_error_string().decode()
    ref_out, ref_lse = api.sparse_attn_fwd(q, k, v, idx, n_split=3)
    torch.cuda.synchronize()
    assert_out_close(out, ref_out.double().cpu().numpy())
    assert_lse_close(lse, ref_lse.double().cpu().numpy())


def test_static_split_rejects_single_piece(cuda_ok):
    q, k, v, idx = _case(1, 8, 16, 2, 64, 8, 1)
    with pytest.raises(SAError, match="n_split"):
        api.sparse_attn_fwd_split_static(q, k, v, idx, n_split=1)


def _two_calls_against_oracle(d, n_split):
    """Two calls in a row with different inputs; the second is compared with
    the fp64 oracle, so a partial left in the shared array by the first call
    (or a fault shared with the workspace path) would show."""
    B, T, Hq, Hkv, K = 1, 120, 16, 1, 100
    for seed in (31, 32):
        q, k, v, idx = _case(B, T, Hq, Hkv, d, K, seed + d)
        rc, out, lse = _static_call(q, k, v, idx, n_split)
        assert rc == _lib.SA_OK, _lib.load().sa_last_error_string().decode()
    torch.cuda.synchronize()
    ro, rl = oracle.sparse_attn(q.cpu(), k.cpu(), v.cpu(), idx.cpu())
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
    api.check_device_status()


@pytest.mark.parametrize("d,n_split", [(128, 4), (64, 2)])
def test_static_split_second_call_matches_oracle(cuda_ok, d, n_split):
    _two_calls_against_oracle(d, n_split)


def test_static_split_on_tensor_core_gather_kernel(cuda_ok):
    # SA_ATTN_PATH is read once per process: run the same check in a fresh
    # process with the tcgen05 gather kernel selected
    code = ("import sys; sys.path.insert(0, 'tests')\n"
            "from test_zz_no_alloc import _two_calls_against_oracle\n"
            "_two_calls_against_oracle(128, 4)\n"
            "print('ok')\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SA_ATTN_PATH="tc")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stderr[-2000:]
