"""Python binding of the pkv C ABI: torch tensors in, raw pointers out.

Argument marshalling only - every step of the path runs in libpkv.so.  Torch
supplies device memory and the current stream.  Names follow include/pkv.h.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Tuple

import torch

from . import _native as N

_DT = {torch.float32: N.PKV_F32, torch.bfloat16: N.PKV_BF16, torch.int8: N.PKV_I8,
       torch.float8_e4m3fn: N.PKV_FP8}


def _dtype_code(dtype: torch.dtype) -> int:
    try:
        return _DT[dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {dtype}") from None


def _dt(t: torch.Tensor) -> int:
    return _dtype_code(t.dtype)


def _ptr(t: Optional[torch.Tensor], dev: Optional[int] = None) -> Optional[int]:
    """Raw address of a contiguous CUDA tensor (on device index dev, if given)."""
    if t is None:
        return None
    i = t.get_device()
    if i < 0:
        raise ValueError("tensor must be on a CUDA device")
    if dev is not None and i != dev:
        raise ValueError(f"tensors on cuda:{dev} and cuda:{i}: all must be on one device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream, dev: Optional[int] = None) -> int:
    """The raw handle of `stream`, by default the current stream of device dev."""
    if stream is None:
        return torch.cuda.current_stream(dev).cuda_stream
    if dev is not None and stream.device.index != dev:
        raise ValueError(f"stream is on {stream.device}, the tensors on cuda:{dev}")
    return stream.cuda_stream


def _device(t: torch.Tensor) -> int:
    """Device index of t; every other tensor of the call must be on it (_ptr)."""
    i = t.get_device()
    if i < 0:
        raise ValueError("tensor must be on a CUDA device")
    return i


def _on(dev: int, fn, *args):
    """Calls the library with dev as the current device: its kernels launch on
    the current device, so memory of another one must never reach them."""
    if torch.cuda.current_device() == dev:
        return fn(*args)
    with torch.cuda.device(dev):
        return fn(*args)


# Shape checks of what the C ABI cannot see: it gets pointers and sizes, so a
# tensor smaller than the sizes passed with it would be read or written past
# its end.  Everything the ABI checks itself (dtypes, supported sizes,
# alignment, workspace size) is left to it.

def _check_cache(k_cache, v_cache, k_scale, v_scale, head_dim: int):
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("k_cache and v_cache must both be [num_blocks, block_size, "
                         "num_kv_heads, head_dim] of one dtype")
    nb, bs, nkv, d = k_cache.shape
    if d != head_dim:
        raise ValueError(f"head_dim {head_dim} of the inputs differs from the cache's {d}")
    for sc in (k_scale, v_scale):
        if sc is not None and (sc.dtype != torch.float32 or sc.numel() != nb * nkv * bs):
            raise ValueError("k_scale and v_scale must be float32 "
                             "[num_blocks, num_kv_heads, block_size]")
    return nb, bs, nkv


def _check_tables(block_tables, context_lens, num_seqs: int) -> None:
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if (block_tables.dim() != 2 or block_tables.shape[0] < num_seqs or
            context_lens.numel() < num_seqs):
        raise ValueError("block_tables must be [num_seqs, max_blocks_per_seq] and "
                         "context_lens [num_seqs]")


def _check_q_out(q, out) -> None:
    if q.dim() != 3:
        raise ValueError("q must be [num_seqs, num_q_heads, head_dim]")
    if out is not None and (out.numel() != q.numel() or out.dtype != q.dtype):
        raise ValueError("out must have q's shape and dtype")


def _check_new(k, v, slot_mapping, num_tokens: int, num_kv_heads: int, head_dim: int) -> None:
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if (k.shape != (num_tokens, num_kv_heads, head_dim) or v.shape != k.shape or
            slot_mapping.numel() < num_tokens):
        raise ValueError("k and v must be [num_tokens, num_kv_heads, head_dim] and "
                         "slot_mapping [num_tokens]")


def _check_flag(err_flag) -> None:
    if err_flag is not None and (err_flag.dtype != torch.int32 or err_flag.numel() < 1):
        raise ValueError("err_flag must be an int32 tensor of at least one element")


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def kv_cache_append(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                    k_cache: torch.Tensor, v_cache: torch.Tensor,
                    k_scale: Optional[torch.Tensor] = None, v_scale: Optional[torch.Tensor] = None,
                    err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """Writes k, v [T, n_kv, d] into the paged caches at slot_mapping [T] (int64).

    Caches are [num_blocks, block_size, n_kv, d]; for int8 and float8_e4m3fn
    caches the fp32 scales are [num_blocks, n_kv, block_size].
    """
    if k.dim() != 3:
        raise ValueError("k and v must be [num_tokens, num_kv_heads, head_dim]")
    T, nkv, d = k.shape
    nb, bs, cache_nkv = _check_cache(k_cache, v_cache, k_scale, v_scale, d)
    if nkv != cache_nkv:
        raise ValueError("k has a different number of kv heads than the cache")
    _check_new(k, v, slot_mapping, T, nkv, d)
    _check_flag(err_flag)
    dev = _device(k)
    rc = _on(dev, N.lib().pkv_kv_cache_append, _ptr(k, dev), _ptr(v, dev), _ptr(slot_mapping, dev),
             T, nkv, d, _dt(k), _ptr(k_cache, dev), _ptr(v_cache, dev), _dt(k_cache), nb, bs,
             _ptr(k_scale, dev), _ptr(v_scale, dev), _ptr(err_flag, dev), _stream(stream, dev))
    N.check(rc, "pkv_kv_cache_append")


def decode_num_splits(num_seqs: int, num_kv_heads: int, head_dim: int, max_context_len: int,
                      cache_dtype: torch.dtype) -> int:
    rc = N.lib().pkv_decode_num_splits(num_seqs, num_kv_heads, head_dim, max_context_len,
                                       _dtype_code(cache_dtype))
    if rc < 0:
        N.check(rc, "pkv_decode_num_splits")
    return rc


def workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                   max_context_len: int, cache_dtype: torch.dtype, num_splits: int = 0) -> int:
    return int(N.lib().pkv_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                          max_context_len, _dtype_code(cache_dtype),
                                          num_splits))


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
    _check_q_out(q, out)
    B, nq, d = q.shape
    nb, bs, nkv = _check_cache(k_cache, v_cache, k_scale, v_scale, d)
    if num_kv_heads is not None and num_kv_heads != nkv:
        raise ValueError("num_kv_heads does not match the cache")
    _check_tables(block_tables, context_lens, B)
    _check_flag(err_flag)
    dev = _device(q)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        need = workspace_size(B, nq, nkv, d, max_context_len, k_cache.dtype, num_splits)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    rc = _on(dev, N.lib().pkv_paged_attention_decode, _ptr(out, dev), _ptr(q, dev), _dt(q),
             _ptr(k_cache, dev), _ptr(v_cache, dev), _dt(k_cache), _ptr(k_scale, dev),
             _ptr(v_scale, dev), _ptr(block_tables, dev), maxb, _ptr(context_lens, dev),
             max_context_len, B, nq, nkv, d, bs, nb, float(softmax_scale), _ptr(workspace, dev),
             _nbytes(workspace), num_splits, _ptr(err_flag, dev), _stream(stream, dev))
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
    _check_q_out(q, out)
    B, nq, d = q.shape
    nb, bs, nkv = _check_cache(k_cache, v_cache, k_scale, v_scale, d)
    _check_tables(block_tables, context_lens, B)
    _check_new(k, v, slot_mapping, B, nkv, d)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k and v must have q's dtype")
    _check_flag(err_flag)
    dev = _device(q)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        need = workspace_size(B, nq, nkv, d, max_context_len, k_cache.dtype, num_splits)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    rc = _on(dev, N.lib().pkv_paged_attention_decode_append, _ptr(out, dev), _ptr(q, dev),
             _ptr(k, dev), _ptr(v, dev), _ptr(slot_mapping, dev), _dt(q), _ptr(k_cache, dev),
             _ptr(v_cache, dev), _dt(k_cache), _ptr(k_scale, dev), _ptr(v_scale, dev),
             _ptr(block_tables, dev), maxb, _ptr(context_lens, dev), max_context_len, B, nq, nkv, d,
             bs, nb, float(softmax_scale), _ptr(workspace, dev), _nbytes(workspace), num_splits,
             _ptr(err_flag, dev), _stream(stream, dev))
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
    _check_q_out(q, out)
    B, nq, d = q.shape
    nb, bs, nkv = _check_cache(k_cache, v_cache, k_scale, v_scale, d)
    _check_tables(block_tables, context_lens, B)
    _check_flag(err_flag)
    dev = _device(q)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    rc = _on(dev, N.lib().pkv_paged_attention_decode_noalloc, _ptr(out, dev), _ptr(q, dev), _dt(q),
             _ptr(k_cache, dev), _ptr(v_cache, dev), _dt(k_cache), _ptr(k_scale, dev),
             _ptr(v_scale, dev), _ptr(block_tables, dev), maxb, _ptr(context_lens, dev),
             max_context_len, B, nq, nkv, d, bs, nb, float(softmax_scale), num_splits,
             _ptr(err_flag, dev), _stream(stream, dev))
    N.check(rc, "pkv_paged_attention_decode_noalloc")
    return out


def shared_prefix_workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                                 head_dim: int, max_context_len: int, prefix_len: int,
                                 cache_dtype: torch.dtype, num_splits: int = 0) -> int:
    return int(N.lib().pkv_shared_prefix_workspace_size(
        num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, prefix_len,
        _dtype_code(cache_dtype), num_splits))


def shared_prefix_plan(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                       max_context_len: int, prefix_len: int, cache_dtype: torch.dtype,
                       num_splits: int = 0) -> Tuple[int, int]:
    """(prefix slices, suffix splits) of a shared-prefix call with these sizes."""
    ps, ss = ctypes.c_int(0), ctypes.c_int(0)
    N.check(N.lib().pkv_shared_prefix_plan(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                           max_context_len, prefix_len,
                                           _dtype_code(cache_dtype), num_splits,
                                           ctypes.byref(ps), ctypes.byref(ss)),
            "pkv_shared_prefix_plan")
    return ps.value, ss.value


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
    _check_q_out(q, out)
    B, nq, d = q.shape
    nb, bs, nkv = _check_cache(k_cache, v_cache, None, None, d)
    _check_tables(block_tables, context_lens, B)
    _check_flag(err_flag)
    dev = _device(q)
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
    rc = _on(dev, N.lib().pkv_paged_attention_decode_shared_prefix, _ptr(out, dev), _ptr(q, dev),
             _dt(q), _ptr(k_cache, dev), _ptr(v_cache, dev), _dt(k_cache), None, None,
             _ptr(block_tables, dev), maxb, _ptr(context_lens, dev), max_context_len, B, nq, nkv, d,
             bs, nb, float(softmax_scale), prefix_len, _ptr(workspace, dev), _nbytes(workspace),
             num_splits, _ptr(err_flag, dev), _stream(stream, dev))
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
    _check_q_out(q, out)
    B, nq, d = q.shape
    nb, bs, nkv = _check_cache(k_cache, v_cache, None, None, d)
    _check_tables(block_tables, context_lens, B)
    _check_new(k, v, slot_mapping, B, nkv, d)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k and v must have q's dtype")
    _check_flag(err_flag)
    dev = _device(q)
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
    rc = _on(dev, N.lib().pkv_paged_attention_decode_shared_prefix_append, _ptr(out, dev),
             _ptr(q, dev), _ptr(k, dev), _ptr(v, dev), _ptr(slot_mapping, dev), _dt(q),
             _ptr(k_cache, dev), _ptr(v_cache, dev), _dt(k_cache), _ptr(block_tables, dev), maxb,
             _ptr(context_lens, dev), max_context_len, B, nq, nkv, d, bs, nb, float(softmax_scale),
             prefix_len, _ptr(workspace, dev), _nbytes(workspace), num_splits, _ptr(err_flag, dev),
             _stream(stream, dev))
    N.check(rc, "pkv_paged_attention_decode_shared_prefix_append")
    return out


def read(src: torch.Tensor, sink: torch.Tensor, stream=None) -> None:
    """Streaming read of all of `src` (HBM read-bandwidth probe; over a buffer
    larger than the L2 it also flushes the L2), XOR-folded into the int32
    device word `sink`."""
    if sink.dtype != torch.int32 or sink.numel() < 1:
        raise ValueError("sink must hold one int32")
    dev = _device(src)
    if _device(sink) != dev:
        raise ValueError("src and sink must be on one device")
    rc = _on(dev, N.lib().pkv_read, _ptr(src, dev), _nbytes(src), _ptr(sink, dev),
             _stream(stream, dev))
    N.check(rc, "pkv_read")


def copy(dst: torch.Tensor, src: torch.Tensor, stream=None) -> None:
    """Streaming device copy (HBM bandwidth probe)."""
    nbytes = _nbytes(src)
    if _nbytes(dst) < nbytes:
        raise ValueError("dst too small")
    dev = _device(dst)
    rc = _on(dev, N.lib().pkv_copy, _ptr(dst, dev), _ptr(src, dev), nbytes,
             _stream(stream, dev))
    N.check(rc, "pkv_copy")
