"""Python binding of the pkv C ABI: torch tensors in, raw pointers out.

Argument marshalling only - every step of the path runs in libpkv.so.  Torch
supplies device memory and the current stream.  Names follow include/pkv.h.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import _native as N

_DT = {torch.float32: N.PKV_F32, torch.bfloat16: N.PKV_BF16, torch.int8: N.PKV_I8,
       torch.float8_e4m3fn: N.PKV_FP8}


def _dt(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if t.device.type != "cuda":
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def kv_cache_append(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                    k_cache: torch.Tensor, v_cache: torch.Tensor,
                    k_scale: Optional[torch.Tensor] = None, v_scale: Optional[torch.Tensor] = None,
                    err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """Writes k, v [T, n_kv, d] into the paged caches at slot_mapping [T] (int64).

    Caches are [num_blocks, block_size, n_kv, d]; for int8 and float8_e4m3fn
    caches the fp32 scales are [num_blocks, n_kv, block_size].
    """
    T, nkv, d = k.shape
    nb, bs = k_cache.shape[0], k_cache.shape[1]
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    rc = N.lib().pkv_kv_cache_append(
        _ptr(k), _ptr(v), _ptr(slot_mapping), T, nkv, d, _dt(k), _ptr(k_cache), _ptr(v_cache),
        _dt(k_cache), nb, bs, _ptr(k_scale), _ptr(v_scale), _ptr(err_flag), _stream(stream))
    N.check(rc, "pkv_kv_cache_append")


def decode_num_splits(num_seqs: int, num_kv_heads: int, head_dim: int, max_context_len: int,
                      cache_dtype: torch.dtype) -> int:
    rc = N.lib().pkv_decode_num_splits(num_seqs, num_kv_heads, head_dim, max_context_len,
                                       _DT[cache_dtype])
    if rc < 0:
        N.check(rc, "pkv_decode_num_splits")
    return rc


def workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                   max_context_len: int, cache_dtype: torch.dtype, num_splits: int = 0) -> int:
    return int(N.lib().pkv_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                          max_context_len, _DT[cache_dtype], num_splits))


def paged_attention_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           block_tables: torch.Tensor, context_lens: torch.Tensor,
                           num_kv_heads: Optional[int] = None,
                           softmax_scale: Optional[float] = None,
                           k_scale: Optional[torch.Tensor] = None,
                           v_scale: Optional[torch.Tensor] = None,
                           max_context_len: Optional[int] = None,
                           out: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
                           err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode attention of q [B, n_q, d] over the paged caches; returns out [B, n_q, d].

    ``max_context_len`` is a host-side upper bound of context_lens (default:
    the block-table capacity).  ``workspace`` (uint8, >= workspace_size bytes)
    is allocated when not given.
    """
    B, nq, d = q.shape
    nb, bs, nkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if num_kv_heads is not None and num_kv_heads != nkv:
        raise ValueError("num_kv_heads does not match the cache")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    cdt = k_cache.dtype
    if workspace is None:
        need = workspace_size(B, nq, nkv, d, max_context_len, cdt, num_splits)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    rc = N.lib().pkv_paged_attention_decode(
        _ptr(out), _ptr(q), _dt(q), _ptr(k_cache), _ptr(v_cache), _dt(k_cache), _ptr(k_scale),
        _ptr(v_scale), _ptr(block_tables), maxb, _ptr(context_lens), max_context_len, B, nq, nkv,
        d, bs, nb, float(softmax_scale), _ptr(workspace), workspace.numel(), num_splits,
        _ptr(err_flag), _stream(stream))
    N.check(rc, "pkv_paged_attention_decode")
    return out


def paged_attention_decode_append(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  slot_mapping: torch.Tensor, k_cache: torch.Tensor,
                                  v_cache: torch.Tensor, block_tables: torch.Tensor,
                                  context_lens: torch.Tensor,
                                  softmax_scale: Optional[float] = None,
                                  k_scale: Optional[torch.Tensor] = None,
                                  v_scale: Optional[torch.Tensor] = None,
                                  max_context_len: Optional[int] = None,
                                  out: Optional[torch.Tensor] = None,
                                  workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
                                  err_flag: Optional[torch.Tensor] = None,
                                  stream=None) -> torch.Tensor:
    """One decode step in one launch: appends each sequence's new token k, v
    [B, n_kv, d] (bf16) at slot_mapping [B] (int64), then attends; the same
    result and cache as kv_cache_append followed by paged_attention_decode when
    slot_mapping[s] is the slot of position context_lens[s] - 1."""
    B, nq, d = q.shape
    nb, bs, nkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    cdt = k_cache.dtype
    if workspace is None:
        need = workspace_size(B, nq, nkv, d, max_context_len, cdt, num_splits)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if k.shape != (B, nkv, d) or v.shape != (B, nkv, d) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k and v must be [num_seqs, num_kv_heads, head_dim] in q's dtype")
    rc = N.lib().pkv_paged_attention_decode_append(
        _ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(slot_mapping), _dt(q), _ptr(k_cache),
        _ptr(v_cache), _dt(k_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables), maxb,
        _ptr(context_lens), max_context_len, B, nq, nkv, d, bs, nb, float(softmax_scale),
        _ptr(workspace), workspace.numel(), num_splits, _ptr(err_flag), _stream(stream))
    N.check(rc, "pkv_paged_attention_decode_append")
    return out


def paged_attention_decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor,
                                   v_cache: torch.Tensor, block_tables: torch.Tensor,
                                   context_lens: torch.Tensor,
                                   softmax_scale: Optional[float] = None,
                                   k_scale: Optional[torch.Tensor] = None,
                                   v_scale: Optional[torch.Tensor] = None,
                                   max_context_len: Optional[int] = None,
                                   out: Optional[torch.Tensor] = None, num_splits: int = 0,
                                   err_flag: Optional[torch.Tensor] = None,
                                   stream=None) -> torch.Tensor:
    """paged_attention_decode for callers that cannot allocate device memory.

    The split-K scratch is the library's fixed 16 MiB device array, so nothing
    is allocated for it; shapes that need more raise PkvError (status -8).
    Calls that overlap on the GPU share that array and race.  ``out`` should be
    passed by such callers (it is only allocated here when omitted).
    """
    B, nq, d = q.shape
    nb, bs, nkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    rc = N.lib().pkv_paged_attention_decode_noalloc(
        _ptr(out), _ptr(q), _dt(q), _ptr(k_cache), _ptr(v_cache), _dt(k_cache), _ptr(k_scale),
        _ptr(v_scale), _ptr(block_tables), maxb, _ptr(context_lens), max_context_len, B, nq, nkv,
        d, bs, nb, float(softmax_scale), num_splits, _ptr(err_flag), _stream(stream))
    N.check(rc, "pkv_paged_attention_decode_noalloc")
    return out


def shared_prefix_workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                                 head_dim: int, max_context_len: int, prefix_len: int,
                                 cache_dtype: torch.dtype, num_splits: int = 0) -> int:
    return int(N.lib().pkv_shared_prefix_workspace_size(
        num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, prefix_len,
        _DT[cache_dtype], num_splits))


def paged_attention_decode_shared_prefix(q: torch.Tensor, k_cache: torch.Tensor,
                                         v_cache: torch.Tensor, block_tables: torch.Tensor,
                                         context_lens: torch.Tensor, prefix_len: int,
                                         softmax_scale: Optional[float] = None,
                                         max_context_len: Optional[int] = None,
                                         out: Optional[torch.Tensor] = None,
                                         workspace: Optional[torch.Tensor] = None,
                                         num_splits: int = 0,
                                         err_flag: Optional[torch.Tensor] = None,
                                         stream=None) -> torch.Tensor:
    """Decode attention for a batch whose sequences share their first
    ``prefix_len`` tokens (same physical blocks, taken from sequence 0's table).
    Same result as paged_attention_decode; the shared blocks are read once per
    KV head for all sequences."""
    B, nq, d = q.shape
    nb, bs, nkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        need = shared_prefix_workspace_size(B, nq, nkv, d, max_context_len, prefix_len,
                                            k_cache.dtype, num_splits)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    rc = N.lib().pkv_paged_attention_decode_shared_prefix(
        _ptr(out), _ptr(q), _dt(q), _ptr(k_cache), _ptr(v_cache), _dt(k_cache), None, None,
        _ptr(block_tables), maxb, _ptr(context_lens), max_context_len, B, nq, nkv, d, bs, nb,
        float(softmax_scale), prefix_len, _ptr(workspace), workspace.numel(), num_splits,
        _ptr(err_flag), _stream(stream))
    N.check(rc, "pkv_paged_attention_decode_shared_prefix")
    return out


def paged_attention_decode_shared_prefix_append(
        q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
        k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
        context_lens: torch.Tensor, prefix_len: int, softmax_scale: Optional[float] = None,
        max_context_len: Optional[int] = None, out: Optional[torch.Tensor] = None,
        workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
        err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """paged_attention_decode_shared_prefix with each sequence's new token k, v
    [B, n_kv, d] appended at slot_mapping [B] in the same call (the token's
    position context_lens[s] - 1 must lie past the shared prefix)."""
    B, nq, d = q.shape
    nb, bs, nkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        need = shared_prefix_workspace_size(B, nq, nkv, d, max_context_len, prefix_len,
                                            k_cache.dtype, num_splits)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if k.shape != (B, nkv, d) or v.shape != (B, nkv, d) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k and v must be [num_seqs, num_kv_heads, head_dim] in q's dtype")
    rc = N.lib().pkv_paged_attention_decode_shared_prefix_append(
        _ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(slot_mapping), _dt(q), _ptr(k_cache),
        _ptr(v_cache), _dt(k_cache), _ptr(block_tables), maxb, _ptr(context_lens),
        max_context_len, B, nq, nkv, d, bs, nb, float(softmax_scale), prefix_len,
        _ptr(workspace), workspace.numel(), num_splits, _ptr(err_flag), _stream(stream))
    N.check(rc, "pkv_paged_attention_decode_shared_prefix_append")
    return out


def copy(dst: torch.Tensor, src: torch.Tensor, stream=None) -> None:
    """Streaming device copy (HBM bandwidth probe)."""
    nbytes = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < nbytes:
        raise ValueError("dst too small")
    N.check(N.lib().pkv_copy(_ptr(dst), _ptr(src), nbytes, _stream(stream)), "pkv_copy")
