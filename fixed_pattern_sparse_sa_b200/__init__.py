"""B200 (sm_100a) causal sparse attention: C-ABI library libsa.so + torch binding.

Importing the package does not load the CUDA library; the first call of an
operation does, and raises if libsa.so is missing (there is no CPU path).
"""
from .api import (SAError, check_device_status, dsa_decode_layers, indexer_topk,  # noqa: F401
                  lse_combine, nsa_fwd, sparse_attn_fwd)

__version__ = "0.1.0"
