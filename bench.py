#!/usr/bin/env python
"""Benchmark of one paged-KV decode step on B200.

A step is the whole hot path over one batch: each sequence's new token is
appended to the cache, then every sequence attends over its context (split-K
plus merge when the planner splits).  By default the step is one call,
``paged_attention_decode_append`` (the append runs inside the decode kernel);
``--unfused`` times ``kv_cache_append`` followed by ``paged_attention_decode``.
Inputs are seeded synthetic tensors shaped like the named workload and
resident in HBM before the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--only]
    python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N
    python bench.py --impl reference      # the CPU oracle, same metric and config
    python bench.py --append              # kv_cache_append: bulk pre-fill and decode step
    python bench.py --swap                # block swap out/in through pinned host memory

Prints one JSON line (rank 0).  The headline workload is the Llama-2-70B-shaped
GQA decode (the largest configuration); unless ``--only`` is given, the
13B-shaped INT8 and the 7B-shaped MHA decodes are measured in the same run and
reported under ``per_workload``.

Timing: W untimed steps, then exactly K steps between a barrier and a device
synchronisation, each step bracketed by its own pair of CUDA events.  Between
steps the L2 is flushed by a streaming read of a buffer twice its size (pkv_read:
loads only, so no dirty line is left for the next step to write back); the
flush sits outside the events.  ``value`` is the KV bytes read by all ranks'
K steps over the max-over-ranks sum of the per-step event times; the median and
minimum per-step times are reported beside the mean.  Multi-GPU runs are
replicas: every rank owns its own batch and block pool (the sequences are
independent), so there is no collective in the data path; the only collectives
are a barrier and max-reductions of the timings.
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
HEADLINE = "llama2-70b-gqa"
COMPANIONS = ("llama2-13b-int8", "llama2-7b-mha")
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--only", action="store_true",
                    help="measure the named workload alone (no per_workload companions)")
    ap.add_argument("--companion-steps", type=int, default=0,
                    help="timed steps of each companion workload (default max(K, 100))")
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-copy-probe", action="store_true",
                    help="skip the same-run HBM copy and read probes")
    ap.add_argument("--no-flush", action="store_true",
                    help="do not flush the L2 between steps")
    ap.add_argument("--no-breakdown", action="store_true",
                    help="skip the per-kernel breakdown of one call")
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
    return ap.parse_args(argv)


# ---------------------------------------------------------------- peaks, clocks

def measured_peaks():
    """HBM GB/s and bf16 TFLOP/s from the generated MEASURED_PEAKS.json,
    else the pool's earlier measurement."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]),
                "bf16_tflops": float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "source": "fallback"}


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clocks_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
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

    def sample_once(self):
        nv = self.nv
        try:
            sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
            reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            power = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
            self.samples.append((sm, reasons, power))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample_once()
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
        if self.ok:  # closing sample: a short region still gets two
            self.sample_once()

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


def kernel_sources(cache_dtype):
    """The source files the decode kernel of this cache format is built from."""
    main = "decode_q8.cu" if cache_dtype in ("i8", "fp8") else "decode.cu"
    return [main, "decode_common.cuh", "decode.cuh", "common.cuh"]


def kernel_source_digest(cache_dtype) -> str:
    h = hashlib.sha256()
    for name in kernel_sources(cache_dtype):
        with open(os.path.join(ROOT, "paged_kv_cache_439_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(wl):
    """DRAM bytes per decode launch of this workload from the committed ncu
    records, or None when none matches it or the kernel's sources changed
    since the capture."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            recs = json.load(f).get("records", [])
    except Exception:
        return None
    digest = kernel_source_digest(wl.cache_dtype)
    for rec in recs:
        if (rec.get("workload") == wl.name and rec.get("block_size") == wl.block_size and
                rec.get("cache_dtype") == wl.cache_dtype and
                rec.get("kernel_sources_sha256_16") == digest):
            return rec
    return None


# ---------------------------------------------------------------- CPU oracle

class OracleArm:
    """The oracle's own paged cache of a workload, filled with the oracle's
    append and decoded with the oracle's gather-then-attend (fp64)."""

    def __init__(self, wl):
        import numpy as np
        import oracle
        self.np, self.oracle, self.wl = np, oracle, wl
        shape = (wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_dim)
        if wl.cache_dtype in ("i8", "fp8"):
            dt = np.int8 if wl.cache_dtype == "i8" else np.uint8
            self.k, self.v = np.zeros(shape, dt), np.zeros(shape, dt)
            sshape = (wl.num_blocks, wl.num_kv_heads, wl.block_size)
            self.ks, self.vs = np.ones(sshape, np.float32), np.ones(sshape, np.float32)
        elif wl.cache_dtype == "bf16":
            self.k, self.v = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
        else:
            self.k, self.v = np.zeros(shape, np.float32), np.zeros(shape, np.float32)

    def _rows(self, x):
        import torch
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(self.np.uint16)
        return x.numpy()

    def _append(self, k, v, slots):
        o, sl = self.oracle, slots.numpy()
        if self.wl.cache_dtype == "i8":
            o.append_int8(k.float().numpy(), sl, self.k, self.ks)
            o.append_int8(v.float().numpy(), sl, self.v, self.vs)
        elif self.wl.cache_dtype == "fp8":
            o.append_fp8(k.float().numpy(), sl, self.k, self.ks)
            o.append_fp8(v.float().numpy(), sl, self.v, self.vs)
        else:
            o.append_rows(self._rows(k), sl, self.k)
            o.append_rows(self._rows(v), sl, self.v)

    def fill(self):
        wl = self.wl
        self._append(wl.prefill_k, wl.prefill_v, wl.prefill_slots)
        self._append(wl.new_k, wl.new_v, wl.new_slots)
        return self

    def decode(self, threads: int = 0):
        np, o, wl = self.np, self.oracle, self.wl
        q = wl.q.float().numpy()
        bt, cl = wl.block_tables.numpy(), wl.context_lens.numpy()
        if wl.cache_dtype == "i8":
            return o.paged_decode_i8(q, self.k, self.v, self.ks, self.vs, bt, cl,
                                     wl.softmax_scale, threads)
        if wl.cache_dtype == "fp8":
            return o.paged_decode_fp8(q, self.k, self.v, self.ks, self.vs, bt, cl,
                                      wl.softmax_scale, threads)
        if wl.cache_dtype == "bf16":
            widen = lambda b: (b.astype(np.uint32) << 16).view(np.float32)
            return o.paged_decode(q, widen(self.k), widen(self.v), bt, cl, wl.softmax_scale,
                                  threads)
        return o.paged_decode(q, self.k, self.v, bt, cl, wl.softmax_scale, threads)


def oracle_sample(name, block_size, budget_s):
    """The first b sequences of the workload in the oracle's own cache, b chosen
    so that one oracle decode of them takes about budget_s (at least one).

    Returns (workload, oracle cache, OpenMP threads)."""
    import oracle
    from paged_kv_cache_439_b200.workloads import make_workload
    one = OracleArm(make_workload(name, block_size=block_size, batch=1)).fill()
    t0 = time.perf_counter()
    one.decode()
    t1 = time.perf_counter() - t0
    cores = oracle.max_threads()
    B = make_workload(name, block_size=block_size).num_seqs
    b = int(max(1, min(B, budget_s / max(t1, 1e-6))))
    wl = make_workload(name, block_size=block_size, batch=b)
    return wl, OracleArm(wl).fill(), cores


def run_cpu_baseline(name, block_size, seconds):
    from paged_kv_cache_439_b200.workloads import make_workload
    wl, oc, cores = oracle_sample(name, block_size, budget_s=min(seconds / 3, 5.0))
    reps, t_total = 0, 0.0
    while t_total < seconds or reps == 0:
        t0 = time.perf_counter()
        oc.decode()
        t_total += time.perf_counter() - t0
        reps += 1
    v = wl.kv_bytes() * reps / t_total / 1e9
    # the same oracle on one thread, over the first sequence alone
    wl1 = make_workload(name, block_size=block_size, batch=1)
    oc1 = OracleArm(wl1).fill()
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
        "config": config_dict(full, args),
        "tokens_per_s_per_layer": round(wl.num_seqs * K / dt, 2),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"each step: oracle decode of the first {wl.num_seqs} of "
                                   f"{full.num_seqs} sequences ({wl.kv_bytes()} KV bytes)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(wl, args, flushed=None):
    lens = wl.context_lens.tolist()
    ctx = f"{lens[0]} each" if len(set(lens)) == 1 else \
        f"{min(lens)}..{max(lens)} (total {sum(lens)})"
    cascade = bool(getattr(args, "cascade", False))
    if flushed is None:
        flushed = not getattr(args, "no_flush", False)
    return {
        "workload": wl.name, "batch": wl.num_seqs, "context_lens": ctx,
        "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
        "head_dim": wl.head_dim, "block_size": wl.block_size, "cache_dtype": wl.cache_dtype,
        "num_blocks": wl.num_blocks,
        "shared_prefix_pass": cascade,
        "step": ("kv_cache_append (1 new token per sequence) + the attention call"
                 if (getattr(args, "unfused", False) or wl.cache_dtype == "f32") else
                 "the attention call with the append fused in (1 new token per sequence "
                 "written inside the decode kernel)"),
        "kv_bytes_per_step": wl.kv_bytes(),
        "l2": l2_note(wl, flushed),
        "parallelism": f"replicas x{getattr(args, 'gpus', 1)} (each rank its own batch and pool)",
    }


def unique_kv_bytes(wl) -> int:
    """Distinct K/V (and scale) bytes a step reads: shared blocks counted once."""
    import torch
    bt = wl.block_tables
    blocks = torch.unique(bt[(bt >= 0) & (bt < wl.num_blocks)]).numel()
    per_row = 2 * wl.head_dim * wl.cache_elem_bytes() + (8 if wl.cache_dtype in ("i8", "fp8")
                                                         else 0)
    return blocks * wl.block_size * wl.num_kv_heads * per_row


def l2_note(wl, flushed: bool):
    """How the timed steps stand to the L2."""
    unique = unique_kv_bytes(wl)
    size = (f"distinct KV {unique // 10**6} MB, "
            f"{'larger than' if unique > L2_BYTES else 'fits'} the 126 MB L2")
    if flushed:
        return (f"{size}; L2 flushed between steps (streaming read of a {2 * L2_BYTES >> 20} "
                f"MiB buffer, outside the per-step events)")
    return f"{size}; not flushed between steps (L2 reuse across steps is part of the number)"


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
    del pk, pv, ps
    return tdt, k_cache, v_cache, k_scale, v_scale, err


class Flusher:
    """Flushes the L2 with a streaming read (pkv_read) of a buffer twice its size."""

    def __init__(self, dev, enabled=True):
        import torch
        import paged_kv_cache_439_b200 as pkv
        self.pkv, self.enabled = pkv, enabled
        self.buf = torch.ones(2 * L2_BYTES, dtype=torch.uint8, device=dev) if enabled else None
        self.sink = torch.zeros(1, dtype=torch.int32, device=dev)

    def __call__(self):
        if self.enabled:
            self.pkv.read(self.buf, self.sink)


def same_run_peaks(dev):
    """The streaming copy (read + write bytes) and the streaming read over
    2 GiB buffers in this process: best of 6 launches after 2 untimed ones."""
    import torch
    import paged_kv_cache_439_b200 as pkv
    nbytes = 2 << 30
    a = torch.ones(nbytes, dtype=torch.uint8, device=dev)
    b = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)

    def best(fn):
        t = 1e9
        for i in range(8):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i >= 2:
                t = min(t, e0.elapsed_time(e1))
        return t

    t_copy = best(lambda: pkv.copy(b, a))
    t_read = best(lambda: pkv.read(a, sink))
    del a, b
    torch.cuda.empty_cache()
    return {"copy_gbs": round(2 * nbytes / (t_copy / 1e3) / 1e9, 1),
            "read_gbs": round(nbytes / (t_read / 1e3) / 1e9, 1),
            "buffers": "2 GiB; copy counts read + write bytes, read counts bytes read"}


def kernel_breakdown(call, flush, dev, reps=20):
    """Device time of each kernel of one call.  The call is captured into a
    CUDA graph (driver API); each of its kernel nodes is re-launched from a
    graph of its own, in the captured order, between CUDA events on one stream
    (L2 flushed before each repetition).  Returns a list of {kernel, ms_mean,
    ms_median}, or {"error": ...} when the bindings are not available."""
    import torch
    try:
        from cuda.bindings import driver as cu
    except Exception as e:  # pragma: no cover - depends on the image
        return {"error": f"cuda-python driver bindings unavailable: {e}"}

    def ok(res, what):
        err = res[0] if isinstance(res, tuple) else res
        if int(err) != 0:
            raise RuntimeError(f"{what}: {err}")
        return res[1:] if isinstance(res, tuple) and len(res) > 1 else None

    graphs, execs = [], []
    try:
        s = torch.cuda.Stream(dev)
        hs = cu.CUstream(s.cuda_stream)
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            ok(cu.cuStreamBeginCapture(
                hs, cu.CUstreamCaptureMode.CU_STREAM_CAPTURE_MODE_RELAXED), "begin capture")
            try:
                call()
            finally:
                (graph,) = ok(cu.cuStreamEndCapture(hs), "end capture")
        graphs.append(graph)
        _, n = ok(cu.cuGraphGetNodes(graph, 0), "node count")
        nodes, _ = ok(cu.cuGraphGetNodes(graph, n), "nodes")
        deps, byid = {}, {}
        v2 = getattr(cu, "cuGraphNodeGetDependencies_v2", None)
        for nd in nodes:
            byid[int(nd)] = nd
            if v2 is not None:
                # with edge data (programmatic launch edges carry some); an
                # upper bound on the count, unused entries come back null
                res = ok(v2(nd, len(nodes)), "deps")
                d = [x for x in res[0] if x is not None and int(x) != 0]
            else:
                _, nd_n = ok(cu.cuGraphNodeGetDependencies(nd, 0), "deps count")
                d = ok(cu.cuGraphNodeGetDependencies(nd, nd_n), "deps")[0] if nd_n else []
            deps[int(nd)] = [int(x) for x in d]
        order, seen = [], set()
        while len(order) < len(nodes):  # the capture of one stream: a chain
            ready = [i for i in byid if i not in seen and all(x in seen for x in deps[i])]
            if not ready:
                raise RuntimeError("capture is not a DAG")
            for i in ready:
                seen.add(i)
                order.append(byid[i])
        names = []
        for nd in order:
            (typ,) = ok(cu.cuGraphNodeGetType(nd), "node type")
            if typ != cu.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
                continue
            (params,) = ok(cu.cuGraphKernelNodeGetParams(nd), "kernel params")
            (g1,) = ok(cu.cuGraphCreate(0), "graph create")
            graphs.append(g1)
            ok(cu.cuGraphAddKernelNode(g1, None, 0, params), "add kernel node")
            (ex,) = ok(cu.cuGraphInstantiate(g1, 0), "instantiate")
            execs.append(ex)
            name = None
            for getter, handle in ((getattr(cu, "cuFuncGetName", None), params.func),
                                   (getattr(cu, "cuKernelGetName", None),
                                    getattr(params, "kern", None))):
                if name or getter is None or handle is None or int(handle) == 0:
                    continue
                try:
                    res = getter(handle)
                    if int(res[0]) == 0:
                        name = res[1].decode() if isinstance(res[1], bytes) else str(res[1])
                except Exception:
                    name = None
            names.append(name or f"kernel {len(names)}")
        times = [[] for _ in execs]
        for _ in range(reps):
            with torch.cuda.stream(s):
                flush()
                evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(execs) + 1)]
                evs[0].record(s)
                for i, ex in enumerate(execs):
                    ok(cu.cuGraphLaunch(ex, hs), "launch")
                    evs[i + 1].record(s)
            s.synchronize()
            for i in range(len(execs)):
                times[i].append(evs[i].elapsed_time(evs[i + 1]))
        return [{"kernel": nm, "ms_mean": round(statistics.mean(t), 5),
                 "ms_median": round(statistics.median(t), 5)} for nm, t in zip(names, times)]
    except Exception as e:
        torch.cuda.synchronize()
        return {"error": repr(e)[:300]}
    finally:
        for ex in execs:
            try:
                cu.cuGraphExecDestroy(ex)
            except Exception:
                pass
        for g in graphs:
            try:
                cu.cuGraphDestroy(g)
            except Exception:
                pass


class StepRunner:
    """One workload's device state and its decode step through the public API."""

    def __init__(self, name, args, dev, rank):
        import torch
        import paged_kv_cache_439_b200 as pkv
        from paged_kv_cache_439_b200 import dist as pdist
        from paged_kv_cache_439_b200.workloads import make_workload, workload_seed
        self.torch, self.pkv, self.dev = torch, pkv, dev
        extra = {"cache_dtype": args.kv_dtype} if args.kv_dtype else {}
        self.wl = wl = make_workload(name, block_size=args.block_size,
                                     data_seed=pdist.replica_seed(workload_seed(name), rank),
                                     **extra)
        (self.tdt, self.k_cache, self.v_cache, self.k_scale, self.v_scale,
         self.err) = device_cache(wl, dev)
        self.q = wl.q.to(dev)
        self.nk, self.nv, self.ns = wl.new_k.to(dev), wl.new_v.to(dev), wl.new_slots.to(dev)
        self.bt, self.cl = wl.block_tables.to(dev), wl.context_lens.to(dev)
        self.max_ctx = wl.max_context_len
        self.prefix_len = int(wl.meta.get("shared_prefix", 0)) if args.cascade else 0
        if args.cascade and self.prefix_len == 0:
            raise SystemExit("--cascade needs a workload with a shared prefix")
        if self.prefix_len:
            # the call's own plan (0 = automatic): the prefix pass fills the
            # suffix decode's last wave, so it splits less than a plain decode
            self.prefix_slices, self.splits = pkv.shared_prefix_plan(
                wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, self.max_ctx,
                self.prefix_len, self.tdt, args.num_splits)
            ws_bytes = pkv.shared_prefix_workspace_size(
                wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, self.max_ctx,
                self.prefix_len, self.tdt, self.splits)
        else:
            self.splits = args.num_splits or pkv.decode_num_splits(
                wl.num_seqs, wl.num_kv_heads, wl.head_dim, self.max_ctx, self.tdt)
            ws_bytes = pkv.workspace_size(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                          wl.head_dim, self.max_ctx, self.tdt, self.splits)
        self.ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(self.q)
        # the append fused into the attention call unless asked otherwise (fp32
        # caches have no fused form)
        self.fused = not args.unfused and wl.cache_dtype != "f32"
        self.launches = ((3 if self.prefix_len else 1 + (1 if self.splits > 1 else 0)) +
                         (0 if self.fused else 1))

    def attend(self, q, bt, cl, out):
        pkv, wl = self.pkv, self.wl
        if self.prefix_len:
            pkv.paged_attention_decode_shared_prefix(
                q, self.k_cache, self.v_cache, bt, cl, self.prefix_len,
                softmax_scale=wl.softmax_scale, max_context_len=self.max_ctx, out=out,
                workspace=self.ws, num_splits=self.splits, err_flag=self.err)
        else:
            pkv.paged_attention_decode(q, self.k_cache, self.v_cache, bt, cl,
                                       softmax_scale=wl.softmax_scale, k_scale=self.k_scale,
                                       v_scale=self.v_scale, max_context_len=self.max_ctx,
                                       out=out, workspace=self.ws, num_splits=self.splits,
                                       err_flag=self.err)

    def attend_append(self, q, k, v, s, bt, cl, out):
        pkv, wl = self.pkv, self.wl
        if self.prefix_len:
            pkv.paged_attention_decode_shared_prefix_append(
                q, k, v, s, self.k_cache, self.v_cache, bt, cl, self.prefix_len,
                softmax_scale=wl.softmax_scale, max_context_len=self.max_ctx, out=out,
                workspace=self.ws, num_splits=self.splits, err_flag=self.err)
        else:
            pkv.paged_attention_decode_append(q, k, v, s, self.k_cache, self.v_cache, bt, cl,
                                              softmax_scale=wl.softmax_scale,
                                              k_scale=self.k_scale, v_scale=self.v_scale,
                                              max_context_len=self.max_ctx, out=out,
                                              workspace=self.ws, num_splits=self.splits,
                                              err_flag=self.err)

    def step_on(self, q, k, v, s, bt, cl, out):
        """One step on the given (device) inputs, through the public API."""
        if not self.fused:
            self.pkv.kv_cache_append(k, v, s, self.k_cache, self.v_cache, self.k_scale,
                                     self.v_scale, err_flag=self.err)
        if self.fused:
            self.attend_append(q, k, v, s, bt, cl, out)
        else:
            self.attend(q, bt, cl, out)

    def step(self):
        self.step_on(self.q, self.nk, self.nv, self.ns, self.bt, self.cl, self.out)

    def attention_call(self):
        """The timed attention call alone (the append is part of it when fused)."""
        if self.fused:
            self.attend_append(self.q, self.nk, self.nv, self.ns, self.bt, self.cl, self.out)
        else:
            self.attend(self.q, self.bt, self.cl, self.out)

    def check_flags(self):
        self.torch.cuda.synchronize()
        f = int(self.err.item())
        if f != 0:
            raise SystemExit(f"{self.wl.name}: device error flag set: {f}")

    def release(self):
        for a in ("k_cache", "v_cache", "k_scale", "v_scale", "ws", "q", "out"):
            setattr(self, a, None)
        self.torch.cuda.empty_cache()


def timed_steps(runner, K, W, flush, world, local):
    """W untimed steps, then exactly K steps between a barrier and a device
    synchronisation, each step (append and attention) between its own CUDA
    events, the L2 flushed before each (outside the events).  Retimed once when
    the clocks show a thermal or hardware slowdown."""
    import torch
    import torch.distributed as dist
    for _ in range(W):
        flush()
        runner.step()
    runner.check_flags()

    def region():
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(local) as cs:
            start.record()
            for i in range(K):
                flush()
                evs[i][0].record()
                runner.step()
                evs[i][1].record()
            end.record()
            torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return start.elapsed_time(end), [a.elapsed_time(b) for a, b in evs], cs.summary()

    region_ms, call_ms, clocks = region()
    remeasured = False
    if ClockSampler.rejected(clocks):
        region_ms, call_ms, clocks = region()
        remeasured = True
    runner.check_flags()
    return region_ms, call_ms, dict(clocks, remeasured=remeasured)


def e2e_overlapped(runner, K, W, world, dev):
    """The same step end to end through the public API: every step copies its
    inputs from pinned host memory (one packed host-to-device copy) and reads
    its output back (one device-to-host copy).  The copies run on a second
    stream with double-buffered device inputs and outputs, so step i + 1's
    input copy and step i - 1's read-back overlap step i's kernel; the timed
    region runs from before the first input copy to the end of the last
    read-back."""
    import torch
    from paged_kv_cache_439_b200 import dist as pdist
    wl = runner.wl
    pieces = [wl.q, wl.new_k, wl.new_v, wl.new_slots, wl.block_tables, wl.context_lens]
    offs, total = [], 0
    for x in pieces:
        offs.append(total)
        total += (x.numel() * x.element_size() + 15) // 16 * 16
    hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()
    for x, o in zip(pieces, offs):
        n = x.numel() * x.element_size()
        hbuf[o:o + n].copy_(x.contiguous().view(-1).view(torch.uint8))
    dbufs, views = [], []
    for _ in range(2):
        d = torch.empty(total, dtype=torch.uint8, device=dev)
        dbufs.append(d)
        views.append([d[o:o + x.numel() * x.element_size()].view(x.dtype).view(x.shape)
                      for x, o in zip(pieces, offs)])
    outs = [torch.empty_like(runner.out) for _ in range(2)]
    houts = [torch.empty(runner.out.shape, dtype=runner.out.dtype).pin_memory()
             for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in pieces)
    d2h = houts[0].numel() * houts[0].element_size()
    main = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)

    def run(n):
        ready = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]
        copy.wait_stream(main)
        with torch.cuda.stream(copy):
            dbufs[0].copy_(hbuf, non_blocking=True)
            ready[0].record(copy)
        for i in range(n):
            b, nb = i % 2, (i + 1) % 2
            main.wait_event(ready[b])
            runner.step_on(*views[b], outs[b])
            used[b].record(main)
            with torch.cuda.stream(copy):
                if i + 1 < n:
                    if i >= 1:
                        copy.wait_event(used[nb])   # step i - 1 is done with buffer nb
                    dbufs[nb].copy_(hbuf, non_blocking=True)
                    ready[nb].record(copy)
                copy.wait_event(used[b])
                houts[b].copy_(outs[b], non_blocking=True)
        main.wait_stream(copy)

    run(W)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    s0.record(main)
    run(K)
    s1.record(main)
    torch.cuda.synchronize()
    runner.check_flags()
    ms = pdist.max_over_ranks(s0.elapsed_time(s1), device=dev)
    return {"value": round(pdist.whole_job_rate(wl.kv_bytes(), K, world, ms), 2),
            "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / K, 5),
            "overlap": "inputs of step i+1 copied in, and outputs of step i-1 read back, on a "
                       "second stream while step i runs (double-buffered)",
            "l2": "steps back to back as a caller runs them: no L2 flush between steps, and "
                  "no per-step events"}


def measure(name, args, dev, K, W, world, rank, local, peaks, flush, want_e2e=True):
    """Times one workload; returns its JSON block (without the run-wide keys)."""
    import torch
    from paged_kv_cache_439_b200 import dist as pdist
    runner = StepRunner(name, args, dev, rank)
    wl = runner.wl
    region_ms, call_ms, clocks = timed_steps(runner, K, W, flush, world, local)
    sum_ms = pdist.max_over_ranks(sum(call_ms), device=dev)
    region_ms = pdist.max_over_ranks(region_ms, device=dev)
    kv = wl.kv_bytes()
    value = pdist.whole_job_rate(kv, K, world, sum_ms)
    mean_ms, med_ms = statistics.mean(call_ms), statistics.median(call_ms)
    # the roofline counts each distinct K/V byte once: with blocks shared
    # between sequences, the logical bytes (value) include re-reads that HBM
    # does not serve
    unique = unique_kv_bytes(wl)
    roof_bytes = unique if unique < kv else kv
    achieved = roof_bytes / (mean_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    rec = traffic_record(wl)
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": rec.get("dram_bytes_per_launch") if rec else None,
            "peak_source": f"{peaks['source']} (hbm_gbs)",
            "decode_ms_mean": round(mean_ms, 5), "decode_ms_median": round(med_ms, 5),
            "decode_ms_min": round(min(call_ms), 5),
            "frac_median": round(roof_bytes / (med_ms / 1e3) / 1e9 / peak, 4)}
    if roof_bytes != kv:
        roof["bytes"] = (f"distinct K/V bytes, {roof_bytes} per call (shared blocks once); the "
                         f"logical {kv} give {kv / (mean_ms / 1e3) / 1e9:.1f} GB/s (value)")
    if peaks.get("read_gbs"):
        roof["frac_of_same_run_read"] = round(achieved / peaks["read_gbs"], 4)
    if peaks.get("copy_gbs"):
        roof["frac_of_same_run_copy"] = round(achieved / peaks["copy_gbs"], 4)
    roof["headline"] = ("frac: achieved over peak (peak_source); the same achieved rate over this "
                        "run's streaming-read probe (the decode only reads K/V) is "
                        "frac_of_same_run_read, over its copy probe (read + write bytes) "
                        "frac_of_same_run_copy")
    if runner.prefix_len:
        roof["kernel"] = ("pkv_paged_attention_decode_shared_prefix" +
                          ("_append" if runner.fused else "") +
                          " (tcgen05 prefix pass + suffix decode + merge)")
    else:
        roof["kernel"] = ("pkv_paged_attention_decode_append (append + decode + split merge)"
                          if runner.fused else "pkv_paged_attention_decode (decode + split merge)")
    ms_per_step = sum_ms / K
    layers = LAYERS.get(wl.name, 1)
    block = {
        "value": round(value, 2), "unit": "GB/s", "steps": K, "warmup": W,
        "ms_per_step": round(ms_per_step, 5), "region_ms": round(region_ms, 4),
        "dtype": {"i8": "int8-kv/bf16-q", "fp8": "fp8e4m3-kv/bf16-q"}.get(wl.cache_dtype,
                                                                       wl.cache_dtype),
        "config": config_dict(wl, args, flushed=flush.enabled),
        "num_splits": runner.splits,
        **({"prefix_slices": runner.prefix_slices} if runner.prefix_len else {}),
        "pct_of_hbm_peak": round(100 * achieved / peak, 1),
        "tokens_per_s_per_layer": round(wl.num_seqs * world / (ms_per_step / 1e3), 1),
        "model_tokens_per_s": round(wl.num_seqs * world / (ms_per_step / 1e3) / layers, 1),
        "model_layers": layers,
        "roofline": roof,
        "clocks": clocks,
        "gpu_launches": K * (runner.launches + (1 if flush.enabled else 0)),
    }
    if runner.prefix_len:
        block["cascade"] = cascade_rooflines(runner, mean_ms, peaks, flush, dev)
    elif not args.no_breakdown:
        block["kernels"] = kernel_breakdown(runner.attention_call, flush, dev)
        runner.check_flags()
    if want_e2e and not args.no_e2e:
        block["e2e"] = e2e_overlapped(runner, K, W, world, dev)
    runner.release()
    return block


def cascade_rooflines(runner, call_ms, peaks, flush, dev):
    """Shared-prefix call: the suffix decode against its unique K/V bytes, the
    tcgen05 prefix pass against its flops and the measured bf16 peak, the
    whole call against the distinct K/V bytes it must read at least once."""
    wl = runner.wl
    P = runner.prefix_len
    rows = wl.num_seqs * wl.group
    elem = wl.cache_elem_bytes()
    suffix_tokens = int((wl.context_lens.to("cpu").long() - P).clamp(min=0).sum().item())
    suffix_bytes = suffix_tokens * wl.num_kv_heads * 2 * wl.head_dim * elem
    prefix_bytes = P * wl.num_kv_heads * 2 * wl.head_dim * elem
    # S = Q K^T (2 rows d flops per token) and O += P V with P as bf16 hi + lo (2 x 2 rows d)
    prefix_flops = 3 * 2 * rows * P * wl.head_dim * wl.num_kv_heads
    unique = unique_kv_bytes(wl)
    out = {"unique_kv_bytes": unique, "suffix_kv_bytes": suffix_bytes,
           "prefix_kv_bytes_once_per_kv_head": prefix_bytes, "prefix_pass_flops": prefix_flops,
           "logical_kv_gbs": round(wl.kv_bytes() / (call_ms / 1e3) / 1e9, 1),
           "call": {"bound": "hbm", "achieved": round(unique / (call_ms / 1e3) / 1e9, 1),
                    "unit": "GB/s", "frac": round(unique / (call_ms / 1e3) / 1e9 /
                                                  peaks["hbm_gbs"], 4)}}
    kb = kernel_breakdown(runner.attention_call, flush, dev)
    runner.check_flags()
    out["kernels"] = kb
    if isinstance(kb, list) and len(kb) == 3:
        def ms_of(tag):
            return next((k["ms_mean"] for k in kb if tag in k["kernel"]), None)
        t_pre, t_merge = ms_of("prefix_kernel"), ms_of("merge_kernel")
        t_suf = next((k["ms_mean"] for k in kb
                      if "prefix_kernel" not in k["kernel"] and "merge_kernel" not in k["kernel"]),
                     None)
    if isinstance(kb, list) and len(kb) == 3 and None not in (t_pre, t_suf, t_merge):
        out["prefix_pass"] = {"bound": "tensor", "achieved": round(prefix_flops / (t_pre / 1e3)
                                                                   / 1e12, 1),
                              "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": round(prefix_flops / (t_pre / 1e3) / 1e12 /
                                            peaks["bf16_tflops"], 4), "ms": t_pre}
        out["suffix_decode"] = {"bound": "hbm", "achieved": round(suffix_bytes / (t_suf / 1e3)
                                                                  / 1e9, 1),
                                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": round(suffix_bytes / (t_suf / 1e3) / 1e9 /
                                              peaks["hbm_gbs"], 4), "ms": t_suf}
        out["merge_ms"] = t_merge
    return out


def run_append(args):
    """Append bandwidth: the workload's pre-fill tokens (up to 65,536) written
    by one kv_cache_append call, against the bytes it must move (K and V rows
    read in the input dtype, written in the cache's, plus the scales of one-byte
    caches), the L2 flushed before every call; and the decode-step append of
    one token per sequence."""
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
    flush = Flusher(dev, enabled=not args.no_flush)

    def timed(fn, reps):
        for _ in range(3):
            flush()
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush()
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return ts

    reps = max(3, min(args.steps, 50))
    t_bulk = timed(lambda: pkv.kv_cache_append(bk, bv, bsl, k_cache, v_cache, ks, vs,
                                               err_flag=err), reps)
    t_step = timed(lambda: pkv.kv_cache_append(nk, nv, ns, k_cache, v_cache, ks, vs,
                                               err_flag=err), reps)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"append kernel flagged {int(err.item())}")
    per_tok = wl.num_kv_heads * wl.head_dim * 2 * (bk.element_size() + wl.cache_elem_bytes())
    if ks is not None:
        per_tok += wl.num_kv_heads * 2 * 4
    peaks = measured_peaks()
    med = statistics.median(t_bulk)
    gbs = T * per_tok / (med * 1e-3) / 1e9
    line = {"metric": "KV append GB/s (bytes read and written by one kv_cache_append call)",
            "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": reps, "warmup": 3,
            "higher_is_better": True,
            "config": {"workload": wl.name, "cache_dtype": wl.cache_dtype, "tokens": T,
                       "bytes_per_token": per_tok, "bytes_per_call": T * per_tok,
                       "l2": "flushed before every call" if flush.enabled else "not flushed"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "peak_source": peaks["source"]},
            "bulk_ms_median": round(med, 4), "bulk_ms_min": round(min(t_bulk), 4),
            "decode_append_us_median": round(statistics.median(t_step) * 1e3, 2),
            "decode_append_tokens": wl.num_seqs}
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

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

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


def main(argv=None):
    args = parse(argv)
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

    from paged_kv_cache_439_b200.workloads import canonical_name
    K, W = args.steps, max(3, args.warmup)
    peaks = measured_peaks()
    if not args.no_copy_probe:
        try:
            peaks.update(same_run_peaks(dev))
        except Exception as e:  # informational only
            peaks["probe_error"] = repr(e)[:200]
    flush = Flusher(dev, enabled=not args.no_flush)

    name = canonical_name(args.workload)
    head = measure(name, args, dev, K, W, world, rank, local, peaks, flush)
    unflushed = None
    if name == "shared-prefix" and flush.enabled:
        # the shared blocks fit the L2: the same steps without the flush as well
        unflushed = measure(name, args, dev, K, W, world, rank, local, peaks,
                            Flusher(dev, enabled=False), want_e2e=False)
    companions = {}
    if not args.only and name == HEADLINE and not args.cascade and not args.kv_dtype:
        Kc = args.companion_steps or max(K, 100)
        for cname in COMPANIONS:
            companions[cname] = measure(cname, args, dev, Kc, W, world, rank, local, peaks,
                                        flush)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(name, args.block_size, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": head["dtype"],
            "data": "synthetic (seeded N(0,1) K/V/q shaped like the workload; no weights)",
            "config": head["config"],
            "num_splits": head["num_splits"],
            **({"prefix_slices": head["prefix_slices"]} if "prefix_slices" in head else {}),
            "pct_of_hbm_peak": head["pct_of_hbm_peak"],
            "tokens_per_s_per_layer": head["tokens_per_s_per_layer"],
            "model_tokens_per_s": head["model_tokens_per_s"],
            "model_layers": head["model_layers"],
            "roofline": head["roofline"],
            "same_run_peaks": {k: peaks[k] for k in ("copy_gbs", "read_gbs", "buffers",
                                                    "probe_error") if k in peaks},
            "cpu_baseline": cpu,
            "e2e": head.get("e2e"),
            "clocks": head["clocks"],
            "gpu_launches": head["gpu_launches"],
            "timing": ("per-step CUDA events around the attention call; value = KV bytes of "
                       "all ranks' K steps / max-over-ranks sum of the per-step times; "
                       "region_ms includes the L2 flushes between steps"),
            "region_ms": head["region_ms"],
        }
        for key in ("kernels", "cascade"):
            if key in head:
                line[key] = head[key]
        if unflushed is not None:
            line["unflushed"] = {k: unflushed[k] for k in (
                "value", "ms_per_step", "roofline", "cascade", "kernels", "config", "clocks")
                if k in unflushed}
        if companions:
            line["per_workload"] = {
                n: {k: b[k] for k in ("value", "unit", "steps", "ms_per_step", "dtype",
                                      "pct_of_hbm_peak", "tokens_per_s_per_layer",
                                      "model_tokens_per_s", "roofline", "e2e", "kernels",
                                      "clocks", "gpu_launches", "config", "num_splits")
                    if k in b}
                for n, b in companions.items()}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
