#!/usr/bin/env python
"""Benchmark of one paged-KV decode step on B200.

A step is the whole hot path over one batch: each sequence's new token is
appended to the cache, then every sequence attends over its context (split-K
plus merge when the planner splits).  By default the step is one call,
``paged_attention_decode_append`` (the append runs inside the decode kernel);
``--unfused`` times ``kv_cache_append`` followed by ``paged_attention_decode``.  Inputs are seeded
synthetic tensors shaped like the named workload and resident in HBM before
the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N
    python bench.py --impl reference      # the CPU oracle, same metric and config
    python bench.py --swap                # block swap out/in through pinned host memory

Prints one JSON line (rank 0).  ``value`` is KV bytes read by the decode
calls of all ranks divided by the max-over-ranks device time of the K timed
steps.  Multi-GPU runs are replicas: every rank owns its own batch and block
pool (the sequences are independent), so there is no collective in the data
path; the only collectives are a barrier and a max-reduction of the timings.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attn KV-read GB/s (% of B200 HBM peak); decode tokens/s per layer"
LAYERS = {"tiny": 1, "llama2-7b-mha": 32, "llama2-70b-gqa": 80, "llama2-13b-int8": 40,
          "shared-prefix": 32}
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama2-7b-mha")
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-copy-probe", action="store_true")
    ap.add_argument("--kv-dtype", choices=["bf16", "i8", "fp8"], default=None,
                    help="override the workload's KV-cache format")
    ap.add_argument("--cascade", action="store_true",
                    help="shared-prefix workload: read the shared blocks once per KV head")
    ap.add_argument("--unfused", action="store_true",
                    help="time the step as two calls (kv_cache_append, then decode) instead of "
                         "the one-launch paged_attention_decode_append")
    ap.add_argument("--append", action="store_true",
                    help="time kv_cache_append: the workload's pre-fill tokens (up to 65,536) "
                         "in one call, and the one-token-per-sequence decode append")
    ap.add_argument("--swap", action="store_true",
                    help="time swapping every sequence's blocks out to pinned host memory and "
                         "back (pkv_copy_blocks) against a plain pinned memcpy of the same bytes")
    return ap.parse_args()


# ---------------------------------------------------------------- peaks, clocks

def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clocks_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(
                        uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h = h
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                power = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((sm, reasons, power))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": "no NVML samples"}
        sms = [s for s, _, _ in self.samples]
        seen = set()
        for _, r, _ in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    seen.add(name)
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(seen), "samples": len(self.samples),
                "power_w_max": round(max(p for _, _, p in self.samples), 1)}

    @staticmethod
    def rejected(summary) -> bool:
        bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
        if bad & set(summary.get("reasons", [])):
            return True
        sm, mx = summary.get("sm_mhz"), summary.get("sm_max_mhz")
        if sm and mx and sm < 0.5 * mx and not summary.get("reasons"):
            return True
        return False


def traffic_record(cache_dtype: str):
    """DRAM bytes per decode launch from the committed ncu summary, or None when
    the decode kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    src = os.path.join(ROOT, "paged_kv_cache_439_b200", "csrc", "decode.cu")
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if rec.get("decode_cu_sha256_16") != digest:
        return None
    return rec


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(name, block_size, budget_s):
    """The first b sequences of the workload in the oracle's own cache, b chosen
    so that one oracle decode of them takes about budget_s (at least one).

    Returns (workload, oracle cache, OpenMP threads)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from pkv_testlib import OracleCache
    from paged_kv_cache_439_b200.workloads import make_workload
    one_wl = make_workload(name, block_size=block_size, batch=1)
    one = OracleCache(one_wl).fill()
    t0 = time.perf_counter()
    one.decode()
    t1 = time.perf_counter() - t0
    cores = oracle.max_threads()
    B = make_workload(name, block_size=block_size).num_seqs
    b = int(max(1, min(B, budget_s / max(t1, 1e-6))))
    wl = make_workload(name, block_size=block_size, batch=b)
    oc = OracleCache(wl).fill()
    return wl, oc, cores


def run_cpu_baseline(name, block_size, seconds):
    wl, oc, cores = oracle_sample(name, block_size, budget_s=min(seconds / 3, 5.0))
    reps, t_total = 0, 0.0
    while t_total < seconds or reps == 0:
        t0 = time.perf_counter()
        oc.decode()
        t_total += time.perf_counter() - t0
        reps += 1
    v = wl.kv_bytes() * reps / t_total / 1e9
    # the same oracle on one thread, over the first sequence alone
    from pkv_testlib import OracleCache
    from paged_kv_cache_439_b200.workloads import make_workload
    wl1 = make_workload(name, block_size=block_size, batch=1)
    oc1 = OracleCache(wl1).fill()
    reps1, t1 = 0, 0.0
    while t1 < min(seconds / 4, 3.0) or reps1 == 0:
        t0 = time.perf_counter()
        oc1.decode(threads=1)
        t1 += time.perf_counter() - t0
        reps1 += 1
    v1 = wl1.kv_bytes() * reps1 / t1 / 1e9
    return {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{name}: oracle decode of the first {wl.num_seqs} sequences "
                      f"({wl.kv_bytes()} KV bytes) x {reps} repetitions, {t_total:.1f} s, "
                      f"fp64, {cores} OpenMP threads",
            "single_thread": {"value": round(v1, 4), "unit": "GB/s",
                              "sample": f"the first sequence ({wl1.kv_bytes()} KV bytes) x "
                                        f"{reps1}, {t1:.1f} s, one thread"}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from paged_kv_cache_439_b200.workloads import make_workload
    full = make_workload(args.workload, block_size=args.block_size)
    K, W = args.steps, args.warmup
    budget = max(0.05, 150.0 / (K + W))
    wl, oc, cores = oracle_sample(args.workload, args.block_size, budget_s=budget)
    for _ in range(W):
        oc.decode()
    t0 = time.perf_counter()
    for _ in range(K):
        oc.decode()
    dt = time.perf_counter() - t0
    value = wl.kv_bytes() * K / dt / 1e9
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": K, "warmup": W, "ms_per_step": round(dt / K * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(full, args, splits=None),
        "tokens_per_s_per_layer": round(wl.num_seqs * K / dt, 2),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"each step: oracle decode of the first {wl.num_seqs} of "
                                   f"{full.num_seqs} sequences ({wl.kv_bytes()} KV bytes)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(wl, args, splits):
    lens = wl.context_lens.tolist()
    ctx = f"{lens[0]} each" if len(set(lens)) == 1 else \
        f"{min(lens)}..{max(lens)} (total {sum(lens)})"
    return {
        "workload": wl.name, "batch": wl.num_seqs, "context_lens": ctx,
        "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
        "head_dim": wl.head_dim, "block_size": wl.block_size, "cache_dtype": wl.cache_dtype,
        "num_blocks": wl.num_blocks, "num_splits": splits,
        "shared_prefix_pass": bool(getattr(args, "cascade", False)),
        "step": ("kv_cache_append (1 new token per sequence) + the attention call"
                 if (getattr(args, "unfused", False) or wl.cache_dtype == "f32") else
                 "the attention call with the append fused in (1 new token per sequence "
                 "written inside the decode kernel)"),
        "kv_bytes_per_step": wl.kv_bytes(),
        "l2": l2_note(wl),
        "parallelism": f"replicas x{args.gpus} (each rank its own batch and pool)",
    }


def l2_note(wl):
    """How the timed steps stand to the L2: the distinct K/V bytes the step reads
    (shared blocks counted once) against the L2 size."""
    import torch
    bt = wl.block_tables
    blocks = torch.unique(bt[(bt >= 0) & (bt < wl.num_blocks)]).numel()
    unique = blocks * wl.block_size * wl.num_kv_heads * wl.head_dim * 2 * wl.cache_elem_bytes()
    if unique > L2_BYTES:
        return (f"inputs larger than L2 (distinct KV {unique // 10**6} MB > 126 MB L2), "
                f"no flush")
    return (f"distinct KV {unique // 10**6} MB fits the 126 MB L2 and is not flushed between "
            f"steps: L2 reuse across steps is part of this workload's number")


# ---------------------------------------------------------------- GPU arm

def device_cache(wl, dev):
    """The workload's paged cache on the device, pre-filled through the C ABI."""
    import torch
    import paged_kv_cache_439_b200 as pkv
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "i8": torch.int8,
           "fp8": torch.float8_e4m3fn}[wl.cache_dtype]
    shape = (wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_dim)
    k_cache = torch.zeros(shape, dtype=torch.uint8 if tdt == torch.float8_e4m3fn else tdt,
                          device=dev).view(tdt)
    v_cache = torch.zeros_like(k_cache)
    k_scale = v_scale = None
    if wl.cache_dtype in ("i8", "fp8"):
        sshape = (wl.num_blocks, wl.num_kv_heads, wl.block_size)
        k_scale = torch.ones(sshape, dtype=torch.float32, device=dev)
        v_scale = torch.ones(sshape, dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pk, pv, ps = (wl.prefill_k.to(dev), wl.prefill_v.to(dev), wl.prefill_slots.to(dev))
    CH = 1 << 16
    for i in range(0, pk.shape[0], CH):
        pkv.kv_cache_append(pk[i:i + CH], pv[i:i + CH], ps[i:i + CH], k_cache, v_cache, k_scale,
                            v_scale, err_flag=err)
    return tdt, k_cache, v_cache, k_scale, v_scale, err


def _event_timer(stream):
    """fn, reps -> mean ms per call on `stream` (three untimed calls first)."""
    import torch

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps
    return timed


def run_append(args):
    """Append bandwidth: the workload's pre-fill tokens (up to 65,536) written
    by one kv_cache_append call, against the bytes it must move (K and V rows
    read in the input dtype, written in the cache's, plus the scales of one-byte
    caches); and the decode-step append of one token per sequence."""
    import torch
    import paged_kv_cache_439_b200 as pkv
    from paged_kv_cache_439_b200.workloads import make_workload, workload_seed
    if int(os.environ.get("RANK", "0")) != 0:
        return
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    extra = {"cache_dtype": args.kv_dtype} if args.kv_dtype else {}
    wl = make_workload(args.workload, block_size=args.block_size,
                       data_seed=workload_seed(args.workload), **extra)
    _, k_cache, v_cache, ks, vs, err = device_cache(wl, dev)
    T = min(wl.prefill_k.shape[0], 1 << 16)
    bk, bv = wl.prefill_k[:T].to(dev), wl.prefill_v[:T].to(dev)
    bsl = wl.prefill_slots[:T].to(dev)
    nk, nv, ns = wl.new_k.to(dev), wl.new_v.to(dev), wl.new_slots.to(dev)
    timed = _event_timer(torch.cuda.current_stream())
    reps = max(1, min(args.steps, 50))
    t_bulk = timed(lambda: pkv.kv_cache_append(bk, bv, bsl, k_cache, v_cache, ks, vs,
                                               err_flag=err), reps)
    t_step = timed(lambda: pkv.kv_cache_append(nk, nv, ns, k_cache, v_cache, ks, vs,
                                               err_flag=err), 10 * reps)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"append kernel flagged {int(err.item())}")
    per_tok = wl.num_kv_heads * wl.head_dim * 2 * (bk.element_size() + wl.cache_elem_bytes())
    if ks is not None:
        per_tok += wl.num_kv_heads * 2 * 4
    peak, peak_src = measured_peak()
    gbs = T * per_tok / (t_bulk * 1e-3) / 1e9
    line = {"metric": "KV append GB/s (bytes read and written by one kv_cache_append call)",
            "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": reps, "warmup": 3,
            "higher_is_better": True,
            "config": {"workload": wl.name, "cache_dtype": wl.cache_dtype, "tokens": T,
                       "bytes_per_token": per_tok},
            "frac_of_hbm_peak": round(gbs / peak, 3), "peak": peak, "peak_source": peak_src,
            "bulk_ms": round(t_bulk, 4),
            "decode_append_us": round(t_step * 1e3, 2), "decode_append_tokens": wl.num_seqs}
    print(json.dumps(line), flush=True)


def run_swap(args):
    """Swap bandwidth: every block of every sequence out to a pinned host pool
    in one pkv_copy_blocks launch, then back in, each timed with CUDA events;
    the plain pinned cudaMemcpyAsync of the same byte count in each direction
    is the link's measured peak."""
    import torch
    import paged_kv_cache_439_b200 as pkv
    from paged_kv_cache_439_b200.workloads import make_workload, workload_seed
    if int(os.environ.get("RANK", "0")) != 0:
        return
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    extra = {"cache_dtype": args.kv_dtype} if args.kv_dtype else {}
    wl = make_workload(args.workload, block_size=args.block_size,
                       data_seed=workload_seed(args.workload), **extra)
    _, k, v, ks, vs, err = device_cache(wl, dev)
    used = list(dict.fromkeys(wl.block_tables[wl.block_tables >= 0].tolist()))
    n = len(used)
    hk = torch.empty((n,) + tuple(k.shape[1:]), dtype=k.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    hks = hvs = None
    if ks is not None:
        hks = torch.empty((n,) + tuple(ks.shape[1:]), dtype=ks.dtype).pin_memory()
        hvs = torch.empty_like(hks).pin_memory()
    out_pairs = torch.tensor([[b, i] for i, b in enumerate(used)], dtype=torch.int32, device=dev)
    in_pairs = out_pairs.flip(1).contiguous()
    nbytes = 2 * (hk.numel() * hk.element_size() + (hks.numel() * 4 if hks is not None else 0))
    flat_dev = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    flat_host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    timed = _event_timer(torch.cuda.current_stream())
    reps = max(1, min(args.steps, 20))
    t_out = timed(lambda: pkv.copy_blocks(hk, hv, k, v, out_pairs, hks, hvs, ks, vs,
                                          err_flag=err), reps)
    t_in = timed(lambda: pkv.copy_blocks(k, v, hk, hv, in_pairs, ks, vs, hks, hvs,
                                         err_flag=err), reps)
    t_d2h = timed(lambda: flat_host.copy_(flat_dev, non_blocking=True), reps)
    t_h2d = timed(lambda: flat_dev.copy_(flat_host, non_blocking=True), reps)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"copy kernel flagged {int(err.item())}")
    gbs = lambda ms: nbytes / (ms * 1e-3) / 1e9
    line = {"metric": "KV block swap GB/s (device<->pinned host, one launch per direction)",
            "value": round(min(gbs(t_out), gbs(t_in)), 2), "unit": "GB/s", "n_gpus": 1,
            "steps": reps, "warmup": 3, "higher_is_better": True,
            "config": {"workload": wl.name, "cache_dtype": wl.cache_dtype, "blocks": n,
                       "bytes_per_direction": nbytes},
            "swap_out_gbs": round(gbs(t_out), 2), "swap_in_gbs": round(gbs(t_in), 2),
            "memcpy_d2h_gbs": round(gbs(t_d2h), 2), "memcpy_h2d_gbs": round(gbs(t_h2d), 2),
            "frac_out": round(t_d2h / t_out, 3), "frac_in": round(t_h2d / t_in, 3)}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.swap:
        run_swap(args)
        return
    if args.append:
        run_append(args)
        return
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)

    import paged_kv_cache_439_b200 as pkv
    from paged_kv_cache_439_b200 import dist as pdist
    from paged_kv_cache_439_b200.workloads import make_workload, workload_seed

    extra = {"cache_dtype": args.kv_dtype} if args.kv_dtype else {}
    wl = make_workload(args.workload, block_size=args.block_size,
                       data_seed=pdist.replica_seed(workload_seed(args.workload), rank), **extra)
    tdt, k_cache, v_cache, k_scale, v_scale, err = device_cache(wl, dev)

    q = wl.q.to(dev)
    nk, nv, ns = wl.new_k.to(dev), wl.new_v.to(dev), wl.new_slots.to(dev)
    bt, cl = wl.block_tables.to(dev), wl.context_lens.to(dev)
    max_ctx = wl.max_context_len
    cache_tdt = tdt
    prefix_len = int(wl.meta.get("shared_prefix", 0)) if args.cascade else 0
    if args.cascade and prefix_len == 0:
        raise SystemExit("--cascade needs a workload with a shared prefix")
    if prefix_len:
        suffix_max = max(max_ctx - prefix_len, 0)
        splits = args.num_splits or pkv.decode_num_splits(wl.num_seqs, wl.num_kv_heads,
                                                           wl.head_dim, suffix_max, cache_tdt)
        ws_bytes = pkv.shared_prefix_workspace_size(wl.num_seqs, wl.num_q_heads,
                                                    wl.num_kv_heads, wl.head_dim, max_ctx,
                                                    prefix_len, cache_tdt, splits)
    else:
        splits = args.num_splits or pkv.decode_num_splits(wl.num_seqs, wl.num_kv_heads,
                                                           wl.head_dim, max_ctx, cache_tdt)
        ws_bytes = pkv.workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                                      max_ctx, cache_tdt, splits)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)

    def attend(qq, btt, cll):
        if prefix_len:
            pkv.paged_attention_decode_shared_prefix(
                qq, k_cache, v_cache, btt, cll, prefix_len, softmax_scale=wl.softmax_scale,
                max_context_len=max_ctx, out=out, workspace=ws, num_splits=splits, err_flag=err)
        else:
            pkv.paged_attention_decode(qq, k_cache, v_cache, btt, cll,
                                       softmax_scale=wl.softmax_scale, k_scale=k_scale,
                                       v_scale=v_scale, max_context_len=max_ctx, out=out,
                                       workspace=ws, num_splits=splits, err_flag=err)

    # the append fused into the attention call unless asked otherwise (fp32
    # caches have no fused form)
    fused = not args.unfused and wl.cache_dtype != "f32"

    def attend_append(qq, kk, vv, ss, btt, cll):
        if prefix_len:
            pkv.paged_attention_decode_shared_prefix_append(
                qq, kk, vv, ss, k_cache, v_cache, btt, cll, prefix_len,
                softmax_scale=wl.softmax_scale, max_context_len=max_ctx, out=out, workspace=ws,
                num_splits=splits, err_flag=err)
        else:
            pkv.paged_attention_decode_append(qq, kk, vv, ss, k_cache, v_cache, btt, cll,
                                              softmax_scale=wl.softmax_scale, k_scale=k_scale,
                                              v_scale=v_scale, max_context_len=max_ctx, out=out,
                                              workspace=ws, num_splits=splits, err_flag=err)

    def step(ev_pair=None):
        if not fused:
            pkv.kv_cache_append(nk, nv, ns, k_cache, v_cache, k_scale, v_scale, err_flag=err)
        if ev_pair is not None:
            ev_pair[0].record()
        if fused:
            attend_append(q, nk, nv, ns, bt, cl)
        else:
            attend(q, bt, cl)
        if ev_pair is not None:
            ev_pair[1].record()

    K, W = args.steps, max(3, args.warmup)
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"device error flag set: {int(err.item())}")

    def timed_region():
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(local) as cs:
            start.record()
            for i in range(K):
                step(evs[i])
            end.record()
            torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        total_ms = start.elapsed_time(end)
        call_ms = [a.elapsed_time(b) for a, b in evs]
        return total_ms, call_ms, cs.summary()

    total_ms, call_ms, clocks = timed_region()
    remeasured = False
    if ClockSampler.rejected(clocks):
        total_ms, call_ms, clocks = timed_region()
        remeasured = True

    max_ms = pdist.max_over_ranks(total_ms, device=dev)
    kv = wl.kv_bytes()
    value = pdist.whole_job_rate(kv, K, world, max_ms)
    decode_ms = statistics.mean(call_ms)
    achieved = kv / (decode_ms / 1e3) / 1e9
    peak, peak_kind = measured_peak()
    rec = traffic_record(wl.cache_dtype)
    traffic = None
    if rec and rec.get("workload") == wl.name and rec.get("block_size") == wl.block_size:
        traffic = rec.get("dram_bytes_per_launch")

    # HBM copy probe in the same process (informational)
    copy_gbs = None
    try:
        if args.no_copy_probe:
            raise RuntimeError("skipped")
        nbytes = 2 << 30
        a = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        b = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        best = 1e9
        for i in range(8):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            pkv.copy(b, a)
            e1.record()
            torch.cuda.synchronize()
            if i >= 2:
                best = min(best, e0.elapsed_time(e1))
        copy_gbs = round(2 * nbytes / (best / 1e3) / 1e9, 1)
        del a, b
    except Exception:
        pass

    # end to end through the public API with pinned host buffers: the step's
    # inputs are packed into one pinned staging buffer (16-byte aligned pieces)
    # and moved with one host-to-device copy; the output comes back with one
    # device-to-host copy
    e2e = None
    if not args.no_e2e:
        pieces = [wl.q, wl.new_k, wl.new_v, wl.new_slots, wl.block_tables, wl.context_lens]
        offs, total = [], 0
        for x in pieces:
            offs.append(total)
            total += (x.numel() * x.element_size() + 15) // 16 * 16
        hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()
        dbuf = torch.empty(total, dtype=torch.uint8, device=dev)
        views = []
        for x, o in zip(pieces, offs):
            n = x.numel() * x.element_size()
            hbuf[o:o + n].copy_(x.contiguous().view(-1).view(torch.uint8))
            views.append(dbuf[o:o + n].view(x.dtype).view(x.shape))
        dq, dk, dv, dsl, dbt, dcl = views
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in pieces)
        d2h = hout.numel() * hout.element_size()

        def e2e_step():
            dbuf.copy_(hbuf, non_blocking=True)
            if fused:
                attend_append(dq, dk, dv, dsl, dbt, dcl)
            else:
                pkv.kv_cache_append(dk, dv, dsl, k_cache, v_cache, k_scale, v_scale,
                                    err_flag=err)
                attend(dq, dbt, dcl)
            hout.copy_(out, non_blocking=True)

        for _ in range(W):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(K):
            e2e_step()
        s1.record()
        torch.cuda.synchronize()
        e2e_ms = pdist.max_over_ranks(s0.elapsed_time(s1), device=dev)
        e2e = {"value": round(pdist.whole_job_rate(kv, K, world, e2e_ms), 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e2e_ms / K, 4)}

    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"device error flag set: {int(err.item())}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(wl.name, args.block_size, args.cpu_seconds)

    if rank == 0:
        ms_per_step = max_ms / K
        layers = LAYERS.get(wl.name, 1)
        launches_per_step = ((3 if prefix_len else 1 + (1 if splits > 1 else 0)) +
                             (0 if fused else 1))
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {"i8": "int8-kv/bf16-q", "fp8": "fp8e4m3-kv/bf16-q"}.get(wl.cache_dtype,
                                                                           wl.cache_dtype),
            "data": "synthetic (seeded N(0,1) K/V/q shaped like the workload; no weights)",
            "config": config_dict(wl, args, splits),
            "pct_of_hbm_peak": round(100 * achieved / peak, 1),
            "tokens_per_s_per_layer": round(wl.num_seqs * world / (ms_per_step / 1e3), 1),
            "model_tokens_per_s": round(wl.num_seqs * world / (ms_per_step / 1e3) / layers, 1),
            "model_layers": layers,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic,
                         "kernel": (("pkv_paged_attention_decode_shared_prefix" +
                                     ("_append" if fused else "") +
                                     " (prefix pass + suffix decode + merge; logical KV bytes)")
                                    if prefix_len else
                                    "pkv_paged_attention_decode_append (append + decode + "
                                    "split merge)" if fused else
                                    "pkv_paged_attention_decode (decode + split merge)"),
                         "peak_source": f"{peak_kind} (hbm_gbs)",
                         "decode_ms_mean": round(decode_ms, 5),
                         "decode_ms_min": round(min(call_ms), 5)},
            "copy_peak_gbs": copy_gbs,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": dict(clocks, remeasured=remeasured),
            "gpu_launches": K * launches_per_step,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
