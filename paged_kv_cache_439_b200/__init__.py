"""Paged-KV decode attention for NVIDIA B200 (sm_100a).

The kernels and their C ABI live in ``libpkv.so`` (``include/pkv.h``); this
package is the thin Python binding plus the seeded workload generator.
"""
from ._native import PkvError, PKV_FLAG_BAD_BLOCK, PKV_FLAG_BAD_SLOT, PKV_FLAG_CTX_RANGE, \
    PKV_FLAG_NEG_CTX, PKV_FLAG_TIMEOUT
from .api import (copy, read, decode_num_splits, kv_cache_append, paged_attention_decode,
                  paged_attention_decode_append, paged_attention_decode_noalloc,
                  paged_attention_decode_shared_prefix,
                  paged_attention_decode_shared_prefix_append,
                  shared_prefix_plan, shared_prefix_workspace_size, workspace_size)
from .block_manager import BlockManager, copy_blocks

__all__ = ["PkvError", "kv_cache_append", "paged_attention_decode",
           "paged_attention_decode_append",
           "paged_attention_decode_noalloc", "paged_attention_decode_shared_prefix",
           "paged_attention_decode_shared_prefix_append",
           "shared_prefix_plan", "shared_prefix_workspace_size", "workspace_size",
           "decode_num_splits", "copy", "read", "BlockManager", "copy_blocks",
           "PKV_FLAG_BAD_BLOCK", "PKV_FLAG_BAD_SLOT",
           "PKV_FLAG_CTX_RANGE", "PKV_FLAG_NEG_CTX", "PKV_FLAG_TIMEOUT"]
