"""CSA2 sparse attention over an FP4 main-KV cache, hand-written for NVIDIA B200 (sm_100a).

The product is libcsa2.so (C ABI, include/csa2.h); `csa2` is its thin Python binding.
"""
from . import csa2  # noqa: F401
from .csa2 import (Csa2Error, index_score_topk, new_workspace, quantize_kv,  # noqa: F401
                   read_device_status, reset_device_status, sparse_attn_decode,
                   sparse_attn_prefill, workspace_bytes)

__all__ = ["csa2", "Csa2Error", "quantize_kv", "index_score_topk", "sparse_attn_decode",
           "sparse_attn_prefill", "workspace_bytes", "new_workspace", "read_device_status",
           "reset_device_status"]
