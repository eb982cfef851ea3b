"""ctypes loader for libsa.so.  Fails loudly when the library is missing."""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsa.so")

# Every symbol declared in include/sa.h.
EXPORTS = (
    "sa_indexer_topk_workspace_size", "sa_indexer_topk",
    "sa_sparse_attn_workspace_size", "sa_sparse_attn_fwd",
    "sa_sparse_attn_fwd_split_static",
    "sa_sparse_attn_bwd_workspace_size", "sa_sparse_attn_bwd",
    "sa_lse_combine",
    "sa_nsa_workspace_size", "sa_nsa_fwd", "sa_nsa_fwd_train",
    "sa_nsa_bwd_workspace_size", "sa_nsa_bwd",
    "sa_full_attn_topk_workspace_size", "sa_full_attn_topk",
    "sa_dsa_decode_layers_workspace_size", "sa_dsa_decode_layers",
    "sa_check_device_status", "sa_last_error_string", "sa_status_string",
    "sa_version", "sa_launch_counter",
    "sa_debug_set_spin_limit", "sa_debug_inject_stall", "sa_debug_exact_recompute_rows",
    "sa_probe_gather",
    "sa_indexer_scores_at", "sa_topk_merge", "sa_index_shard",
)

SA_OK = 0
STATUS = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED",
          3: "SA_ERR_WORKSPACE", 4: "SA_ERR_CUDA", 5: "SA_ERR_DEVICE_ASSERT",
          6: "SA_ERR_TIMEOUT"}
SA_ERR_DEVICE_ASSERT = 5
SA_ERR_TIMEOUT = 6


class SAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class sa_pattern(ctypes.Structure):
    _fields_ = [("window", ctypes.c_int32), ("dilated", ctypes.c_int32)]


class sa_dsa_layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q", "k", "v", "q_idx", "k_idx", "w", "out", "lse")]


_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """Load libsa.so (built in-tree).  Raises if it is missing: there is no
    fallback implementation of any operation."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libsa.so not found at {LIB_PATH}; build it with "
                "`python -m fixed_pattern_sparse_sa_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                            ctypes.c_size_t, ctypes.c_float)
        sig = {
            "sa_indexer_topk_workspace_size": (SZ, [I, I, I, I, I, I, I]),
            "sa_indexer_topk": (I, [P, P, P, I, I, I, I, I, I64, I, I, P, P, P, SZ, P]),
            "sa_sparse_attn_workspace_size": (SZ, [I, I, I, I, I]),
            "sa_sparse_attn_fwd": (I, [P, P, P, I, I, I, I, I, I, I64, P, I, I, P, P, P, P,
                                       F, I, P, P, P, P, P, SZ, P]),
            "sa_sparse_attn_fwd_split_static": (I, [P, P, P, I, I, I, I, I, I, I64, P, I, I,
                                                    F, I, P, P, P]),
            "sa_lse_combine": (I, [P, P, I, I64, I, P, P, P]),
            "sa_sparse_attn_bwd_workspace_size": (SZ, [I, I, I]),
            "sa_sparse_attn_bwd": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I64, P, I, I, F, P, P, P, P, SZ, P]),
            "sa_nsa_workspace_size": (SZ, [I, I, I, I, I, I, I, I, I]),
            "sa_nsa_fwd": (I, [P, P, P, P, I, I, I, I, I, I, I, I, I, I, F, P, P, P, P, SZ, P]),
            "sa_nsa_fwd_train": (I, [P, P, P, P, I, I, I, I, I, I, I, I, I, I, F, P, P, P, P, P, SZ, P]),
            "sa_nsa_bwd_workspace_size": (SZ, [I, I, I, I, I, I, I, I, I]),
            "sa_full_attn_topk_workspace_size": (SZ, [I, I, I, I, I, I, I]),
            "sa_full_attn_topk": (I, [P, P, P, I, I, I, I, I, F, I, I, P, P, P, P, SZ, P]),
            "sa_nsa_bwd": (I, [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, F, P, P, P, P,
                               P, SZ, P]),
            "sa_dsa_decode_layers_workspace_size": (SZ, [I, I, I, I, I, I, I, I, I, I]),
            "sa_dsa_decode_layers": (I, [ctypes.c_char_p, I, P, I, I, I, I, I, I, I, I, I64,
                                         I, I, F, I, P, P, SZ, P]),
            "sa_check_device_status": (I, [P]),
            "sa_last_error_string": (ctypes.c_char_p, []),
            "sa_status_string": (ctypes.c_char_p, [I]),
            "sa_version": (I, []),
            "sa_launch_counter": (ctypes.c_uint64, []),
            "sa_debug_set_spin_limit": (I, [ctypes.c_long]),
            "sa_debug_inject_stall": (I, [I]),
            "sa_debug_exact_recompute_rows": (I64, []),
            "sa_probe_gather": (I, [P, I64, I, I, I, I, I, P, P]),
            "sa_indexer_scores_at": (I, [P, P, P, I, I, I, I, I, P, I, P, P]),
            "sa_topk_merge": (I, [P, P, P, I, I64, I, I, I, I64, P, P, P]),
            "sa_index_shard": (I, [P, I64, I64, I64, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def check(status: int, what: str):
    if status != SA_OK:
        msg = load().sa_last_error_string().decode(errors="replace")
        raise SAError(status, f"{what}: {msg}")
