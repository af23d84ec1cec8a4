"""CSA2 sparse attention over an FP4 main-KV cache, hand-written for NVIDIA B200 (sm_100a).

The product is libcsa2.so (C ABI, include/csa2.h); `csa2` is its thin Python binding and `cp`
the context-parallel orchestration of a Full layer over torch.distributed.
"""
from . import cp, csa2  # noqa: F401
from .csa2 import (Csa2Error, attn_merge_partials, cache_export, cache_import,  # noqa: F401
                   cache_record_bytes, index_score_topk, new_workspace, quantize_kv,
                   read_device_status, reset_device_status, sparse_attn_decode,
                   sparse_attn_decode_partial, sparse_attn_prefill, workspace_bytes)

__all__ = ["csa2", "cp", "Csa2Error", "quantize_kv", "index_score_topk", "sparse_attn_decode",
           "sparse_attn_prefill", "sparse_attn_decode_partial", "attn_merge_partials",
           "workspace_bytes", "new_workspace", "read_device_status", "reset_device_status",
           "cache_record_bytes", "cache_export", "cache_import"]
