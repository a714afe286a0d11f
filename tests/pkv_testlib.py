"""Shared helpers for the parity tests.

Both sides start from the same seeded workload (paged_kv_cache_439_b200.workloads)
and each builds its own paged cache with its own append: the CUDA path through
the C ABI, the oracle through oracle/.  Nothing computed by one side is fed to
the other.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_439_b200.workloads import Workload

# Tolerances (per element, allclose form): bf16/int8 caches |d| <= 2e-3 + 1e-2 |ref|;
# fp32 caches |d| <= 1e-4 * max(1, |ref|).
TOL_BF16 = (2e-3, 1e-2)
TOL_F32 = (1e-4, 1e-4)

BF16_NAN = 0x7FC0


def tol_for(wl: Workload):
    return TOL_F32 if wl.cache_dtype == "f32" else TOL_BF16


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """Exact bf16 -> fp32 widening of raw uint16 bit patterns."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def host_rows(x: torch.Tensor) -> np.ndarray:
    """Append input rows as numpy: bf16 as raw uint16 bits, fp32 as float32."""
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view(np.uint16)
    return x.numpy()


# ---------------------------------------------------------------- oracle side

class OracleCache:
    """The oracle's own paged cache, filled with the oracle's append."""

    def __init__(self, wl: Workload):
        self.wl = wl
        shape = (wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_dim)
        if wl.cache_dtype in ("i8", "fp8"):
            dt = np.int8 if wl.cache_dtype == "i8" else np.uint8
            self.k = np.full(shape, 127, dt)
            self.v = np.full(shape, 127, dt)
            sshape = (wl.num_blocks, wl.num_kv_heads, wl.block_size)
            self.ks = np.full(sshape, np.nan, np.float32)
            self.vs = np.full(sshape, np.nan, np.float32)
        elif wl.cache_dtype == "bf16":
            self.k = np.full(shape, BF16_NAN, np.uint16)
            self.v = np.full(shape, BF16_NAN, np.uint16)
        else:
            self.k = np.full(shape, np.nan, np.float32)
            self.v = np.full(shape, np.nan, np.float32)

    def append(self, k: torch.Tensor, v: torch.Tensor, slots: torch.Tensor) -> None:
        sl = slots.numpy()
        if self.wl.cache_dtype == "i8":
            kf = k.float().numpy()
            vf = v.float().numpy()
            oracle.append_int8(kf, sl, self.k, self.ks)
            oracle.append_int8(vf, sl, self.v, self.vs)
        elif self.wl.cache_dtype == "fp8":
            oracle.append_fp8(k.float().numpy(), sl, self.k, self.ks)
            oracle.append_fp8(v.float().numpy(), sl, self.v, self.vs)
        else:
            oracle.append_rows(host_rows(k), sl, self.k)
            oracle.append_rows(host_rows(v), sl, self.v)

    def fill(self) -> "OracleCache":
        self.append(self.wl.prefill_k, self.wl.prefill_v, self.wl.prefill_slots)
        self.append(self.wl.new_k, self.wl.new_v, self.wl.new_slots)
        return self

    def decode(self, threads: int = 0, block_tables=None) -> np.ndarray:
        wl = self.wl
        q = wl.q.float().numpy()
        bt = (wl.block_tables if block_tables is None else block_tables).numpy()
        cl = wl.context_lens.numpy()
        if wl.cache_dtype == "i8":
            return oracle.paged_decode_i8(q, self.k, self.v, self.ks, self.vs, bt, cl,
                                          wl.softmax_scale, threads)
        if wl.cache_dtype == "fp8":
            return oracle.paged_decode_fp8(q, self.k, self.v, self.ks, self.vs, bt, cl,
                                           wl.softmax_scale, threads)
        if wl.cache_dtype == "bf16":
            return oracle.paged_decode(q, widen_bf16(self.k), widen_bf16(self.v), bt, cl,
                                       wl.softmax_scale, threads)
        return oracle.paged_decode(q, self.k, self.v, bt, cl, wl.softmax_scale, threads)


# ---------------------------------------------------------------- CUDA side

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "i8": torch.int8,
             "fp8": torch.float8_e4m3fn}


class GpuCache:
    """The CUDA path's paged cache on the device, filled through the C ABI."""

    def __init__(self, wl: Workload, device="cuda"):
        import paged_kv_cache_439_b200 as pkv
        self.pkv = pkv
        self.wl = wl
        self.device = device
        shape = (wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_dim)
        dt = _TORCH_DT[wl.cache_dtype]
        if wl.cache_dtype in ("i8", "fp8"):
            self.k = torch.full(shape, 127, dtype=torch.int8, device=device).view(dt)
            self.v = torch.full(shape, 127, dtype=torch.int8, device=device).view(dt)
            sshape = (wl.num_blocks, wl.num_kv_heads, wl.block_size)
            self.ks = torch.full(sshape, float("nan"), dtype=torch.float32, device=device)
            self.vs = torch.full(sshape, float("nan"), dtype=torch.float32, device=device)
        else:
            self.k = torch.full(shape, float("nan"), dtype=dt, device=device)
            self.v = torch.full(shape, float("nan"), dtype=dt, device=device)
            self.ks = self.vs = None
        self.err = torch.zeros(1, dtype=torch.int32, device=device)

    def append(self, k, v, slots) -> None:
        if k.shape[0] == 0:
            return
        self.pkv.kv_cache_append(k.to(self.device), v.to(self.device), slots.to(self.device),
                                 self.k, self.v, self.ks, self.vs, err_flag=self.err)

    def fill(self) -> "GpuCache":
        wl = self.wl
        self.append(wl.prefill_k, wl.prefill_v, wl.prefill_slots)
        self.append(wl.new_k, wl.new_v, wl.new_slots)
        return self

    def decode(self, num_splits: int = 0, block_tables=None, context_lens=None,
               max_context_len=None) -> torch.Tensor:
        wl = self.wl
        bt = (wl.block_tables if block_tables is None else block_tables).to(self.device)
        cl = (wl.context_lens if context_lens is None else context_lens).to(self.device)
        mcl = wl.max_context_len if max_context_len is None else max_context_len
        return self.pkv.paged_attention_decode(
            wl.q.to(self.device), self.k, self.v, bt, cl, softmax_scale=wl.softmax_scale,
            k_scale=self.ks, v_scale=self.vs, max_context_len=mcl, num_splits=num_splits,
            err_flag=self.err)

    def flags(self) -> int:
        return int(self.err.item())


# ---------------------------------------------------------------- comparison

def compare(got: torch.Tensor, ref: np.ndarray, tol) -> dict:
    atol, rtol = tol
    g = got.float().cpu().numpy().astype(np.float64)
    d = np.abs(g - ref)
    bound = atol + rtol * np.abs(ref)
    worst = np.unravel_index(np.argmax(d - bound), d.shape) if d.size else None
    return {
        "ok": bool(np.isfinite(g).all() and (d <= bound).all()),
        "max_abs": float(d.max()) if d.size else 0.0,
        "max_rel": float((d / np.maximum(np.abs(ref), 1e-6)).max()) if d.size else 0.0,
        "worst": worst,
        "finite": bool(np.isfinite(g).all()),
    }


def assert_close(got: torch.Tensor, ref: np.ndarray, tol, what=""):
    r = compare(got, ref, tol)
    assert r["ok"], f"{what}: {r}"
    return r


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a tensor (NaN-safe exact comparison)."""
    t = t.cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def oracle_bits(wl: Workload, arr: np.ndarray) -> np.ndarray:
    if arr.dtype == np.uint16:
        return arr.view(np.int16)
    if arr.dtype == np.float32:
        return arr.view(np.int32)
    return arr
