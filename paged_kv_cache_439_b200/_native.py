"""ctypes loader for libpkv.so (the CUDA kernels and their C ABI, include/pkv.h).

There is no fallback: if the library is missing or does not load, every call
raises.  Build it with ``python -m paged_kv_cache_439_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpkv.so")

PKV_F32, PKV_BF16, PKV_I8, PKV_FP8 = 0, 1, 2, 3

PKV_FLAG_BAD_BLOCK = 1
PKV_FLAG_BAD_SLOT = 2
PKV_FLAG_CTX_RANGE = 4
PKV_FLAG_NEG_CTX = 8
PKV_FLAG_TIMEOUT = 16

PKV_ERR_SCRATCH_LIMIT = -8
PKV_ERR_NO_BLOCKS = -9
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024

# exported symbol -> (restype, argtypes); mirrors include/pkv.h
_vp, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "pkv_kv_cache_append": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _i, _i, _i, _vp, _vp,
                                 _vp, _vp]),
    "pkv_decode_num_splits": (_i, [_i, _i, _i, _i, _i]),
    "pkv_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "pkv_paged_attention_decode": (_i, [_vp, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _i, _vp, _i,
                                        _i, _i, _i, _i, _i, _i, _f, _vp, _sz, _i, _vp, _vp]),
    "pkv_paged_attention_decode_append": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _i, _vp,
                                               _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i,
                                               _f, _vp, _sz, _i, _vp, _vp]),
    "pkv_paged_attention_decode_shared_prefix_append": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _vp,
                                                             _vp, _i, _vp, _i, _vp, _i, _i,
                                                             _i, _i, _i, _i, _i, _f, _i, _vp,
                                                             _sz, _i, _vp, _vp]),
    "pkv_paged_attention_decode_noalloc": (_i, [_vp, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _i,
                                                _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp,
                                                _vp]),
    "pkv_shared_prefix_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "pkv_shared_prefix_plan": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_i),
                                    ctypes.POINTER(_i)]),
    "pkv_paged_attention_decode_shared_prefix": (_i, [_vp, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp,
                                                      _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                                                      _i, _vp, _sz, _i, _vp, _vp]),
    "pkv_copy": (_i, [_vp, _vp, _sz, _vp]),
    "pkv_read": (_i, [_vp, _sz, _vp, _vp]),
    "pkv_copy_blocks": (_i, [_vp, _vp, _vp, _vp, _sz, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp, _i,
                             _vp, _vp]),
    "pkv_bm_create": (_i, [_i, _i, ctypes.POINTER(ctypes.c_void_p)]),
    "pkv_bm_destroy": (None, [_vp]),
    "pkv_bm_num_free": (_i, [_vp]),
    "pkv_bm_ref_count": (_i, [_vp, ctypes.c_int32]),
    "pkv_bm_add_sequence": (_i, [_vp, ctypes.c_int64]),
    "pkv_bm_fork": (_i, [_vp, ctypes.c_int64, ctypes.c_int64]),
    "pkv_bm_blocks_needed": (_i, [_vp, ctypes.c_int64, _i]),
    "pkv_bm_reserve": (_i, [_vp, ctypes.c_int64, _i, _vp, _vp, ctypes.POINTER(_i)]),
    "pkv_bm_free": (_i, [_vp, ctypes.c_int64]),
    "pkv_bm_seq_len": (_i, [_vp, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64),
                            ctypes.POINTER(_i)]),
    "pkv_bm_block_tables": (_i, [_vp, _vp, _i, _i, _vp, _vp]),
    "pkv_bm_swap_out": (_i, [_vp, _vp, ctypes.c_int64, _vp, _i, ctypes.POINTER(_i)]),
    "pkv_bm_swap_in": (_i, [_vp, _vp, ctypes.c_int64, _vp, _i, ctypes.POINTER(_i)]),
    "pkv_strerror": (ctypes.c_char_p, [_i]),
    "pkv_version": (_i, []),
}

_lock = threading.Lock()
_lib = None


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} (status {status})")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(
                        f"libpkv.so not found at {LIB_PATH}; build it with "
                        "`python -m paged_kv_cache_439_b200.build`")
                handle = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    fn = getattr(handle, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = handle
    return _lib


def strerror(status: int) -> str:
    return lib().pkv_strerror(status).decode()


def check(status: int, what: str) -> None:
    if status != 0:
        raise PkvError(status, what)
