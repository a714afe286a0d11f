"""CPU oracle for paged-KV decode attention (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
the two share no code.

The arithmetic lives in ``oracle.c`` (fp64 attention, fp32 quantiser), built
with gcc into ``liboracle.so`` beside this file; this module only marshals
numpy arrays into it.  ``brute`` holds a pure-Python restatement for tiny
inputs.  Each function cites the passage it follows in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, library_path

__all__ = [
    "kv_cache_bytes",
    "append_rows",
    "quantize_row",
    "append_int8",
    "gather",
    "paged_decode",
    "paged_decode_i8",
    "max_threads",
    "e4m3_decode",
    "e4m3_encode",
    "quantize_row_fp8",
    "append_fp8",
    "paged_decode_fp8",
    "copy_blocks",
]

_LIB = None

_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_u64 = ctypes.c_uint64
_vp = ctypes.c_void_p
_dbl = ctypes.c_double


def _lib():
    global _LIB
    if _LIB is None:
        path = build_oracle()
        lib = ctypes.CDLL(path)
        lib.oracle_kv_cache_bytes.restype = _u64
        lib.oracle_kv_cache_bytes.argtypes = [_u64] * 6
        lib.oracle_append_rows.restype = _i32
        lib.oracle_append_rows.argtypes = [_vp, _vp, _i64, _i64, _vp, _i64, _i64]
        lib.oracle_quantize_row.restype = None
        lib.oracle_quantize_row.argtypes = [_vp, _i32, _vp, _vp]
        lib.oracle_append_int8.restype = _i32
        lib.oracle_append_int8.argtypes = [_vp, _vp, _i64, _i32, _i32, _vp, _vp, _i64, _i64]
        lib.oracle_gather_f32.restype = _i32
        lib.oracle_gather_f32.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32]
        lib.oracle_paged_decode_f32.restype = _i32
        lib.oracle_paged_decode_f32.argtypes = [_vp] * 5 + [_i32, _vp] + [_i32] * 6 + [_dbl, _i32]
        lib.oracle_paged_decode_i8.restype = _i32
        lib.oracle_paged_decode_i8.argtypes = [_vp] * 7 + [_i32, _vp] + [_i32] * 6 + [_dbl, _i32]
        lib.oracle_e4m3_decode.restype = _dbl
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_quantize_row_fp8.restype = None
        lib.oracle_quantize_row_fp8.argtypes = [_vp, _i32, _vp, _vp]
        lib.oracle_append_fp8.restype = _i32
        lib.oracle_append_fp8.argtypes = [_vp, _vp, _i64, _i32, _i32, _vp, _vp, _i64, _i64]
        lib.oracle_paged_decode_fp8.restype = _i32
        lib.oracle_paged_decode_fp8.argtypes = [_vp] * 7 + [_i32, _vp] + [_i32] * 6 + [_dbl, _i32]
        lib.oracle_copy_blocks.restype = _i32
        lib.oracle_copy_blocks.argtypes = [_vp, _vp, _i64, _i32, _i32, _vp, _i32]
        lib.oracle_max_threads.restype = _i32
        lib.oracle_max_threads.argtypes = []
        _LIB = lib
    return _LIB


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(_vp)


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what} returned {rc}")


def max_threads() -> int:
    return int(_lib().oracle_max_threads())


def kv_cache_bytes(batch, seq_len, num_layers, num_kv_heads, head_dim, dtype_bytes) -> int:
    """KV-cache size in bytes (GPUYard §2 formula; mlqm.cn §1)."""
    return int(_lib().oracle_kv_cache_bytes(batch, seq_len, num_layers, num_kv_heads, head_dim,
                                            dtype_bytes))


def append_rows(x: np.ndarray, slot_mapping: np.ndarray, cache: np.ndarray) -> None:
    """Copy token rows into their slots, in place on ``cache``.

    x: [T, n_kv, d] (any dtype); cache: [num_blocks, block_size, n_kv, d], same
    dtype.  Negative slots are skipped.
    """
    assert x.dtype == cache.dtype and x.shape[1:] == cache.shape[2:]
    assert cache.flags.c_contiguous
    xb, xp = _c(x, x.dtype)
    sm, sp = _c(slot_mapping, np.int64)
    row_bytes = x.dtype.itemsize * int(np.prod(x.shape[1:]))
    rc = _lib().oracle_append_rows(xp, sp, x.shape[0], row_bytes, cache.ctypes.data_as(_vp),
                                   cache.shape[0], cache.shape[1])
    _check(rc, "oracle_append_rows")


def quantize_row(x: np.ndarray):
    """INT8 quantisation of one fp32 row (mlqm.cn §4).  Returns (codes, scale)."""
    xb, xp = _c(x, np.float32)
    codes = np.zeros(xb.shape[0], dtype=np.int8)
    scale = np.zeros(1, dtype=np.float32)
    _lib().oracle_quantize_row(xp, xb.shape[0], codes.ctypes.data_as(_vp), scale.ctypes.data_as(_vp))
    return codes, scale[0]


def append_int8(x: np.ndarray, slot_mapping: np.ndarray, codes: np.ndarray, scale: np.ndarray) -> None:
    """Quantising append, in place.

    x: fp32-valued [T, n_kv, d]; codes: int8 [num_blocks, block_size, n_kv, d];
    scale: fp32 [num_blocks, n_kv, block_size].
    """
    xb, xp = _c(x, np.float32)
    sm, sp = _c(slot_mapping, np.int64)
    assert codes.dtype == np.int8 and codes.flags.c_contiguous
    assert scale.dtype == np.float32 and scale.flags.c_contiguous
    nb, bs, nkv, d = codes.shape
    assert scale.shape == (nb, nkv, bs) and xb.shape[1:] == (nkv, d)
    rc = _lib().oracle_append_int8(xp, sp, xb.shape[0], nkv, d, codes.ctypes.data_as(_vp),
                                   scale.ctypes.data_as(_vp), nb, bs)
    _check(rc, "oracle_append_int8")


def gather(cache: np.ndarray, table_row: np.ndarray, ctx: int) -> np.ndarray:
    """Contiguous fp64 K (or V) rows [ctx, n_kv, d] of one sequence."""
    cb, cp = _c(cache, np.float32)
    tb, tp = _c(table_row, np.int32)
    nb, bs, nkv, d = cb.shape
    out = np.zeros((max(ctx, 0), nkv, d), dtype=np.float64)
    rc = _lib().oracle_gather_f32(out.ctypes.data_as(_vp), cp, tp, ctx, nkv, d, bs, nb)
    _check(rc, "oracle_gather_f32")
    return out


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, softmax_scale, threads=0):
    """fp64 paged decode attention over fp32-valued caches.

    q: [B, n_q, d]; caches [num_blocks, block_size, n_kv, d]; block_tables int32
    [B, max_blocks]; context_lens int32 [B].  Returns fp64 [B, n_q, d].
    """
    qb, qp = _c(q, np.float32)
    kb, kp = _c(k_cache, np.float32)
    vb, vp = _c(v_cache, np.float32)
    bt, btp = _c(block_tables, np.int32)
    cl, clp = _c(context_lens, np.int32)
    B, nq, d = qb.shape
    nb, bs, nkv, d2 = kb.shape
    assert d == d2 and vb.shape == kb.shape and bt.shape[0] == B and cl.shape == (B,)
    out = np.zeros((B, nq, d), dtype=np.float64)
    rc = _lib().oracle_paged_decode_f32(out.ctypes.data_as(_vp), qp, kp, vp, btp, bt.shape[1], clp,
                                        B, nq, nkv, d, bs, nb, float(softmax_scale), int(threads))
    _check(rc, "oracle_paged_decode_f32")
    return out


def paged_decode_i8(q, k_codes, v_codes, k_scale, v_scale, block_tables, context_lens,
                    softmax_scale, threads=0):
    """fp64 paged decode attention over an INT8 cache (dequantised code / scale)."""
    qb, qp = _c(q, np.float32)
    kb, kp = _c(k_codes, np.int8)
    vb, vp = _c(v_codes, np.int8)
    ks, ksp = _c(k_scale, np.float32)
    vs, vsp = _c(v_scale, np.float32)
    bt, btp = _c(block_tables, np.int32)
    cl, clp = _c(context_lens, np.int32)
    B, nq, d = qb.shape
    nb, bs, nkv, d2 = kb.shape
    assert d == d2 and vb.shape == kb.shape and ks.shape == (nb, nkv, bs) == vs.shape
    out = np.zeros((B, nq, d), dtype=np.float64)
    rc = _lib().oracle_paged_decode_i8(out.ctypes.data_as(_vp), qp, kp, vp, ksp, vsp, btp,
                                       bt.shape[1], clp, B, nq, nkv, d, bs, nb,
                                       float(softmax_scale), int(threads))
    _check(rc, "oracle_paged_decode_i8")
    return out


def e4m3_decode(code: int) -> float:
    """Value of an E4M3 code (OCP FP8 definition)."""
    return float(_lib().oracle_e4m3_decode(int(code) & 0xFF))


def e4m3_encode(y: float) -> int:
    """Nearest E4M3 code, ties to even, saturating at +-448."""
    return int(_lib().oracle_e4m3_encode(float(y)))


def quantize_row_fp8(x: np.ndarray):
    """FP8 quantisation of one fp32 row.  Returns (codes uint8, scale)."""
    xb, xp = _c(x, np.float32)
    codes = np.zeros(xb.shape[0], dtype=np.uint8)
    scale = np.zeros(1, dtype=np.float32)
    _lib().oracle_quantize_row_fp8(xp, xb.shape[0], codes.ctypes.data_as(_vp),
                                   scale.ctypes.data_as(_vp))
    return codes, scale[0]


def append_fp8(x: np.ndarray, slot_mapping: np.ndarray, codes: np.ndarray, scale: np.ndarray) -> None:
    """FP8 quantising append, in place (layouts as append_int8, codes uint8)."""
    xb, xp = _c(x, np.float32)
    sm, sp = _c(slot_mapping, np.int64)
    assert codes.dtype == np.uint8 and codes.flags.c_contiguous
    assert scale.dtype == np.float32 and scale.flags.c_contiguous
    nb, bs, nkv, d = codes.shape
    assert scale.shape == (nb, nkv, bs) and xb.shape[1:] == (nkv, d)
    rc = _lib().oracle_append_fp8(xp, sp, xb.shape[0], nkv, d, codes.ctypes.data_as(_vp),
                                  scale.ctypes.data_as(_vp), nb, bs)
    _check(rc, "oracle_append_fp8")


def paged_decode_fp8(q, k_codes, v_codes, k_scale, v_scale, block_tables, context_lens,
                     softmax_scale, threads=0):
    """fp64 paged decode attention over an FP8 cache (dequantised E4M3(code) / scale)."""
    qb, qp = _c(q, np.float32)
    kb, kp = _c(k_codes, np.uint8)
    vb, vp = _c(v_codes, np.uint8)
    ks, ksp = _c(k_scale, np.float32)
    vs, vsp = _c(v_scale, np.float32)
    bt, btp = _c(block_tables, np.int32)
    cl, clp = _c(context_lens, np.int32)
    B, nq, d = qb.shape
    nb, bs, nkv, d2 = kb.shape
    assert d == d2 and vb.shape == kb.shape and ks.shape == (nb, nkv, bs) == vs.shape
    out = np.zeros((B, nq, d), dtype=np.float64)
    rc = _lib().oracle_paged_decode_fp8(out.ctypes.data_as(_vp), qp, kp, vp, ksp, vsp, btp,
                                        bt.shape[1], clp, B, nq, nkv, d, bs, nb,
                                        float(softmax_scale), int(threads))
    _check(rc, "oracle_paged_decode_fp8")
    return out


def copy_blocks(dst: np.ndarray, src: np.ndarray, pairs: np.ndarray) -> None:
    """dst[pairs[i, 1]] = src[pairs[i, 0]] for whole blocks (first axis), in place."""
    assert dst.dtype == src.dtype and dst.shape[1:] == src.shape[1:] and dst.flags.c_contiguous
    sb, sp = _c(src, src.dtype)
    pb, pp = _c(pairs, np.int32)
    block_bytes = src.dtype.itemsize * int(np.prod(src.shape[1:]))
    rc = _lib().oracle_copy_blocks(dst.ctypes.data_as(_vp), sp, block_bytes, dst.shape[0],
                                   src.shape[0], pp, pb.shape[0])
    _check(rc, "oracle_copy_blocks")
