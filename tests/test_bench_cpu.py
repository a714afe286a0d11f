"""The benchmark's CPU legs: the reference arm (the oracle timed on the host)
and the CPU baseline, on the tiny workload.  They need no GPU, so the JSON
contract of those lines is checked here."""
import importlib.util
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("bench_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _run(*args, env=None):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=600, cwd=ROOT,
                          env={**os.environ, **(env or {})})


def test_reference_arm_prints_one_contract_line():
    r = _run("--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 1
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny" and "l2" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    r = _run("--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0",
             env={"RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_cpu_baseline_reports_threads_and_one_thread():
    bench = _bench_module()
    cb = bench.run_cpu_baseline("tiny", None, 0.2)
    assert cb["kind"] == "oracle" and cb["unit"] == "GB/s" and cb["value"] > 0
    assert cb["cores"] >= 1 and "tiny" in cb["sample"]
    st = cb["single_thread"]
    assert st["value"] > 0 and st["unit"] == "GB/s" and "one thread" in st["sample"]


def test_l2_note_counts_shared_blocks_once():
    bench = _bench_module()
    from paged_kv_cache_439_b200.workloads import make_custom
    shared = make_custom("l2-shared", [300, 300, 300], 4, 2, 64, 16, "bf16", seed=9,
                         shared_prefix=256)
    own = make_custom("l2-own", [300, 300, 300], 4, 2, 64, 16, "bf16", seed=9)
    per_block = 16 * 2 * 64 * 2 * 2
    n_shared = len(set(shared.block_tables[shared.block_tables >= 0].tolist()))
    n_own = len(set(own.block_tables[own.block_tables >= 0].tolist()))
    assert n_shared < n_own
    assert f"distinct KV {n_shared * per_block // 10**6} MB" in bench.l2_note(shared, False)
    assert "fits the 126 MB L2" in bench.l2_note(own, False)
    assert "not flushed" in bench.l2_note(own, False)
    assert "flushed between steps" in bench.l2_note(own, True)
    assert bench.unique_kv_bytes(shared) == n_shared * per_block


def test_bench_oracle_arm_matches_the_test_oracle_cache():
    """The bench's CPU legs build the oracle's cache themselves (they do not
    import the test helpers); on the same workload they give the same output."""
    import numpy as np
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from pkv_testlib import OracleCache
    from paged_kv_cache_439_b200.workloads import make_custom, make_workload
    bench = _bench_module()
    for wl in (make_workload("tiny"),
               make_custom("arm-i8", [40, 300], 8, 2, 64, 16, "i8", seed=3, outlier_prob=0.01),
               make_custom("arm-bf16", [17, 100], 8, 4, 128, 16, "bf16", seed=4)):
        a = bench.OracleArm(wl).fill().decode()
        b = OracleCache(wl).fill().decode()
        assert np.array_equal(a, b)


def test_reference_config_equals_the_gpu_arm_config_keys():
    """Both arms describe the workload with the same config (no planner output in it)."""
    bench = _bench_module()
    from paged_kv_cache_439_b200.workloads import make_workload
    args = bench.parse(["--workload", "tiny"])
    c = bench.config_dict(make_workload("tiny"), args)
    assert "num_splits" not in c and c["workload"] == "tiny"
    assert c == bench.config_dict(make_workload("tiny"), args, flushed=True)
    assert bench.parse([]).workload == "llama2-70b-gqa"


def test_traffic_record_is_used_only_for_the_sources_it_was_captured_on():
    """A committed ncu traffic record reaches the bench line only while the
    decode kernel's sources still hash to the digest stored with it."""
    from types import SimpleNamespace
    b = _bench_module()
    recs = json.load(open(os.path.join(ROOT, "profiles", "decode_traffic.json")))["records"]
    assert recs
    for rec in recs:
        wl = SimpleNamespace(name=rec["workload"], block_size=rec["block_size"],
                             cache_dtype=rec["cache_dtype"])
        assert rec["kernel_sources"] == b.kernel_sources(rec["cache_dtype"])
        b.kernel_source_digest = lambda dt, d=rec["kernel_sources_sha256_16"]: d
        assert b.traffic_record(wl) == rec
        b.kernel_source_digest = lambda dt: "0" * 16      # the sources changed
        assert b.traffic_record(wl) is None
        # traffic within 1% of the algorithmic bytes: no re-reads
        assert 0.98 < rec["traffic_over_algorithmic"] < 1.02
