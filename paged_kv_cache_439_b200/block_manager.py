"""Python binding of the host block manager and the block copier (include/pkv.h).

Marshalling only: the bookkeeping runs in libpkv.so (C++), the copies in its
copy kernel.
"""
from __future__ import annotations

import ctypes
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

from . import _native as N
from .api import _on, _ptr, _stream


class BlockManager:
    """Block ids of one pool: allocation on demand, ref counts, fork,
    copy-on-write and swap bookkeeping."""

    def __init__(self, num_blocks: int, block_size: int):
        h = ctypes.c_void_p()
        N.check(N.lib().pkv_bm_create(num_blocks, block_size, ctypes.byref(h)), "pkv_bm_create")
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self) -> None:
        if self._h:
            N.lib().pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover - interpreter shutdown order
        try:
            self.close()
        except Exception:
            pass

    @property
    def num_free(self) -> int:
        return N.lib().pkv_bm_num_free(self._h)

    def ref_count(self, block: int) -> int:
        r = N.lib().pkv_bm_ref_count(self._h, block)
        if r < 0:
            N.check(r, "pkv_bm_ref_count")
        return r

    def add_sequence(self, seq_id: int) -> None:
        N.check(N.lib().pkv_bm_add_sequence(self._h, seq_id), "pkv_bm_add_sequence")

    def fork(self, parent: int, child: int) -> None:
        N.check(N.lib().pkv_bm_fork(self._h, parent, child), "pkv_bm_fork")

    def blocks_needed(self, seq_id: int, num_tokens: int) -> int:
        r = N.lib().pkv_bm_blocks_needed(self._h, seq_id, num_tokens)
        if r < 0:
            N.check(r, "pkv_bm_blocks_needed")
        return r

    def reserve(self, seq_id: int, num_tokens: int) -> Tuple[np.ndarray, Optional[Tuple[int, int]]]:
        """Slots of the next num_tokens tokens, and the copy-on-write pair if any."""
        slots = np.zeros(max(num_tokens, 1), dtype=np.int64)
        cow = np.zeros(2, dtype=np.int32)
        n = ctypes.c_int(0)
        N.check(N.lib().pkv_bm_reserve(self._h, seq_id, num_tokens,
                                       slots.ctypes.data_as(ctypes.c_void_p),
                                       cow.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)),
                "pkv_bm_reserve")
        return slots[:num_tokens], (int(cow[0]), int(cow[1])) if n.value else None

    def free(self, seq_id: int) -> None:
        N.check(N.lib().pkv_bm_free(self._h, seq_id), "pkv_bm_free")

    def seq_len(self, seq_id: int) -> Tuple[int, int]:
        ln = ctypes.c_int64(0)
        nb = ctypes.c_int(0)
        N.check(N.lib().pkv_bm_seq_len(self._h, seq_id, ctypes.byref(ln), ctypes.byref(nb)),
                "pkv_bm_seq_len")
        return ln.value, nb.value

    def block_tables(self, seq_ids: Sequence[int], max_blocks_per_seq: int):
        ids = np.asarray(seq_ids, dtype=np.int64)
        tables = np.zeros((len(ids), max_blocks_per_seq), dtype=np.int32)
        lens = np.zeros(len(ids), dtype=np.int32)
        N.check(N.lib().pkv_bm_block_tables(self._h, ids.ctypes.data_as(ctypes.c_void_p), len(ids),
                                            max_blocks_per_seq,
                                            tables.ctypes.data_as(ctypes.c_void_p),
                                            lens.ctypes.data_as(ctypes.c_void_p)),
                "pkv_bm_block_tables")
        return tables, lens

    def _move(self, fn, other: "BlockManager", seq_id: int, capacity: int) -> np.ndarray:
        pairs = np.zeros((max(capacity, 1), 2), dtype=np.int32)
        n = ctypes.c_int(0)
        N.check(fn(self._h, other._h, seq_id, pairs.ctypes.data_as(ctypes.c_void_p), capacity,
                   ctypes.byref(n)), "pkv_bm_swap")
        return pairs[:n.value]

    def swap_out(self, host: "BlockManager", seq_id: int) -> np.ndarray:
        """(device block, host block) pairs; the sequence now lives in `host`."""
        return self._move(N.lib().pkv_bm_swap_out, host, seq_id, self.num_blocks)

    def swap_in(self, device: "BlockManager", seq_id: int) -> np.ndarray:
        """(host block, device block) pairs; the sequence now lives in `device`.
        Call on the host-pool manager."""
        return self._move(N.lib().pkv_bm_swap_in, device, seq_id, self.num_blocks)


def _any_ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    """Device tensors, or page-locked host tensors the device can address."""
    if t is None:
        return None
    if t.device.type == "cuda":
        return _ptr(t)
    if not t.is_pinned():
        raise ValueError("host pools must be page-locked (pin_memory())")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def copy_blocks(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor,
                src_v: torch.Tensor, pairs: torch.Tensor,
                dst_k_scale: Optional[torch.Tensor] = None,
                dst_v_scale: Optional[torch.Tensor] = None,
                src_k_scale: Optional[torch.Tensor] = None,
                src_v_scale: Optional[torch.Tensor] = None,
                err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """Copies block pairs[i, 0] of the source pool to block pairs[i, 1] of the
    destination pool (K, V and optional scales).  `pairs` is a device int32
    tensor [n, 2]; pools are device tensors or pinned host tensors."""
    # the library is given one block size and one block count per pool: every
    # tensor of a pool must agree with them, or a copy would run past its end
    if dst_v.shape != dst_k.shape or src_v.shape != src_k.shape or dst_k.dim() < 2:
        raise ValueError("K and V of a pool must have one shape [num_blocks, ...]")
    block_bytes = _block_bytes(src_k)
    if _block_bytes(dst_k) != block_bytes:
        raise ValueError("source and destination blocks differ in size")
    scales = (dst_k_scale, dst_v_scale, src_k_scale, src_v_scale)
    sbytes = 0
    if any(t is not None for t in scales):
        if any(t is None for t in scales):
            raise ValueError("give all four scale pools or none")
        if (dst_v_scale.shape != dst_k_scale.shape or src_v_scale.shape != src_k_scale.shape or
                dst_k_scale.shape[0] != dst_k.shape[0] or src_k_scale.shape[0] != src_k.shape[0]):
            raise ValueError("scale pools must be [num_blocks, ...] like their caches")
        sbytes = _block_bytes(src_k_scale)
        if _block_bytes(dst_k_scale) != sbytes:
            raise ValueError("source and destination scale blocks differ in size")
    if pairs.dtype != torch.int32 or pairs.device.type != "cuda":
        raise TypeError("pairs must be an int32 CUDA tensor")
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [num_pairs, 2]")
    dev = pairs.get_device()
    for t in (dst_k, dst_v, src_k, src_v, err_flag) + scales:
        if t is not None and t.device.type == "cuda" and t.get_device() != dev:
            raise ValueError("device pools, pairs and err_flag must be on one device")
    rc = _on(dev, N.lib().pkv_copy_blocks,
             _any_ptr(dst_k), _any_ptr(dst_v), _any_ptr(src_k), _any_ptr(src_v), block_bytes,
             dst_k.shape[0], src_k.shape[0], _any_ptr(dst_k_scale), _any_ptr(dst_v_scale),
             _any_ptr(src_k_scale), _any_ptr(src_v_scale), sbytes, _ptr(pairs), pairs.shape[0],
             _ptr(err_flag), _stream(stream, dev))
    N.check(rc, "pkv_copy_blocks")


def _block_bytes(pool: torch.Tensor) -> int:
    return math.prod(pool.shape[1:]) * pool.element_size()
