"""CPU checks of the C-ABI boundary: libsa.so loads, exports every symbol
declared in include/sa.h, and rejects bad arguments on the host before any
device work (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from fixed_pattern_sparse_sa_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _header_functions():
    src = open(os.path.join(ROOT, "include", "sa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", src)))


def test_header_and_binding_agree():
    assert _header_functions() == sorted(_lib.EXPORTS)


def test_every_header_symbol_is_exported(lib):
    for name in _header_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.sa_version() == 100
    assert lib.sa_status_string(0) == b"SA_OK"
    assert lib.sa_status_string(5) == b"SA_ERR_DEVICE_ASSERT"
    assert lib.sa_status_string(6) == b"SA_ERR_TIMEOUT"
    assert lib.sa_status_string(99) == b"SA_ERR_UNKNOWN"


def test_workspace_queries(lib):
    # indexer scratch: B * rows-per-chunk * row-length int32 scores, rounded
    n = lib.sa_indexer_topk_workspace_size(1, 512, 512, 2, 32, 64, 32)
    assert n > 0 and n % 256 == 0
    assert lib.sa_sparse_attn_workspace_size(2, 3, 4, 64, 1) == 0
    # partials + lse (384 B rounded to 512) + one merge ticket per row (96 B rounded to 256)
    assert lib.sa_sparse_attn_workspace_size(2, 3, 4, 64, 4) == 4 * 24 * 64 * 4 + 512 + 256
    assert lib.sa_nsa_workspace_size(1, 1024, 16, 1, 64, 32, 16, 64, 16) > 0
    assert lib.sa_indexer_topk_workspace_size(0, 1, 1, 2, 32, 1, 0) == 0
    # NSA backward: compressed rows, their fp32 gradients, D terms, block lists
    assert lib.sa_nsa_bwd_workspace_size(1, 1024, 16, 1, 64, 32, 16, 64, 16) > 0
    assert lib.sa_nsa_bwd_workspace_size(1, 1024, 16, 1, 64, 32, 16, 0, 16) == 0
    # exact indexer: fp32 layer output + lse + one chunk of dense scores (<= 1 GiB)
    full = lib.sa_full_attn_topk_workspace_size(1, 65536, 16, 1, 128, 1024, 128)
    rows = 65536 * 16
    assert (1 << 30) < full <= rows * 128 * 4 + rows * 4 + (1 << 30) + 1024


def test_indexer_workspace_is_chunked_under_one_gib(lib):
    # the prefill indexer processes its query rows in chunks sized so one
    # chunk's sample, thresholds and candidate lists stay within 1 GiB: the
    # workspace grows with the rows until that cap and stays under it after
    # (longer rows mean longer lists, so fewer rows per chunk).  Beside the
    # chunk, prefill-shaped calls keep one copy of the query operand with the
    # weights folded in: B*Tq*Hi*di bytes plus B*Tq*Hi int32 weights.
    def cap(B, T, Hi=16, di=64):
        return (1 << 30) * 1.01 + B * T * Hi * (di + 4) + 1024
    sizes = [lib.sa_indexer_topk_workspace_size(1, t, t, 16, 64, 2048, 0)
             for t in (1024, 4096, 16384, 65536, 131072)]
    assert all(a < b for a, b in zip(sizes[:3], sizes[1:4]))
    assert all(s <= cap(1, t) for s, t in zip(sizes, (1024, 4096, 16384, 65536, 131072)))
    assert min(sizes[3:]) > 0.9 * (1 << 30)
    assert lib.sa_indexer_topk_workspace_size(2, 65536, 65536, 16, 64, 2048, 0) <= cap(2, 65536)
    # decode-shaped calls (one query row per sequence) need far less
    assert lib.sa_indexer_topk_workspace_size(32, 1, 131072, 16, 64, 2048, 0) < sizes[-1] // 100


def test_host_validation_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: rejected first
    # n_split < 1
    assert lib.sa_lse_combine(fake, fake, 0, 4, 64, fake, None, None) == 1
    # unsupported head dim
    assert lib.sa_lse_combine(fake, fake, 2, 4, 96, fake, None, None) == 2
    assert b"head dim" in lib.sa_last_error_string()
    # misaligned pointer
    assert lib.sa_lse_combine(ctypes.c_void_p((1 << 20) + 4), fake, 2, 4, 64, fake, None, None) == 1
    # unsupported indexer head count
    assert lib.sa_indexer_topk(fake, fake, fake, 1, 8, 8, 3, 32, 0, 4, 0, fake, None,
                               fake, 1 << 20, None) == 2
    # query positions beyond the keys
    assert lib.sa_indexer_topk(fake, fake, fake, 1, 8, 8, 2, 32, 1, 4, 0, fake, None,
                               fake, 1 << 20, None) == 1
    # workspace too small
    assert lib.sa_indexer_topk(fake, fake, fake, 1, 8, 8, 2, 32, 0, 4, 0, fake, None,
                               fake, 16, None) == 3
    # pattern must start with F
    arr = (_lib.sa_dsa_layer * 1)()
    assert lib.sa_dsa_decode_layers(b"S", 1, arr, 1, 1, 8, 16, 1, 128, 8, 64, 7, 4, 0,
                                    0.1, 1, None, fake, 1 << 30, None) == 1
    assert b"first layer" in lib.sa_last_error_string()
    # NSA: sel_topk too large
    assert lib.sa_nsa_fwd(fake, fake, fake, fake, 1, 64, 16, 1, 64, 32, 16, 64, 33, 512,
                          0.1, fake, None, None, fake, 1 << 30, None) == 2
    # NSA training forward: the saved branch outputs are required
    assert lib.sa_nsa_fwd_train(fake, fake, fake, fake, 1, 64, 16, 1, 64, 32, 16, 64, 16, 512,
                                0.1, fake, fake, fake, None, fake, 1 << 30, None) == 1
    # NSA backward: head dim, a missing saved tensor, workspace too small
    assert lib.sa_nsa_bwd(fake, fake, fake, fake, fake, fake, fake, fake, 1, 64, 16, 1, 96, 32, 16,
                          64, 16, 512, 0.1, fake, fake, fake, fake, fake, 1 << 30, None) == 2
    assert lib.sa_nsa_bwd(fake, fake, fake, fake, fake, None, fake, fake, 1, 64, 16, 1, 64, 32, 16,
                          64, 16, 512, 0.1, fake, fake, fake, fake, fake, 1 << 30, None) == 1
    assert lib.sa_nsa_bwd(fake, fake, fake, fake, fake, fake, fake, fake, 1, 64, 16, 1, 64, 32, 16,
                          64, 16, 512, 0.1, fake, fake, fake, fake, fake, 64, None) == 3
    # exact indexer from a full layer: Hq not a multiple of Hkv, head dim, no set size, workspace
    assert lib.sa_full_attn_topk(fake, fake, fake, 1, 64, 6, 4, 64, 0.1, 8, 4, None, None, fake,
                                 fake, 1 << 30, None) == 1
    assert lib.sa_full_attn_topk(fake, fake, fake, 1, 64, 4, 1, 96, 0.1, 8, 4, None, None, fake,
                                 fake, 1 << 30, None) == 2
    assert lib.sa_full_attn_topk(fake, fake, fake, 1, 64, 4, 1, 64, 0.1, 0, 0, None, None, fake,
                                 fake, 1 << 30, None) == 1
    assert lib.sa_full_attn_topk(fake, fake, fake, 1, 64, 4, 1, 64, 0.1, 8, 4, None, None, fake,
                                 fake, 64, None) == 3
    # attention: Hq not a multiple of Hkv
    assert lib.sa_sparse_attn_fwd(fake, fake, fake, 1, 4, 4, 3, 2, 64, 0, fake, 1, 4, None,
                                  None, None, None, 0.1, 1, fake, None, None, None, None, 0,
                                  None) == 1


def test_static_split_rejects_wrapping_sizes(lib):
    # n_split * B * Tq * Hq * (d + 1) * 4 must not wrap around size_t and
    # slip under the 8 MiB limit: each product is checked before anything is
    # enqueued (the pointers are never dereferenced)
    fake = ctypes.c_void_p(1 << 20)
    big = (1 << 31) - 1
    for B, Tq, Hq, n_split in [(big, big, big, big), (1, 1 << 20, 1 << 20, 1 << 24), (4, 4, 16, 2 ** 30)]:
        rc = lib.sa_sparse_attn_fwd_split_static(fake, fake, fake, B, Tq, 1 << 20, Hq, 1, 128, 0,
                                                 fake, 1, 8, 0.1, n_split, fake, None, None)
        assert rc == 3, (B, Tq, Hq, n_split)
        assert b"built-in" in lib.sa_last_error_string()


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.load()
