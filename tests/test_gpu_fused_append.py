"""One-launch decode step (append fused into the decode kernel) against the
two-call path and the oracle.

The fused call must leave the cache exactly as kv_cache_append does (codes and
scales bit for bit) and produce the same output as kv_cache_append followed by
paged_attention_decode, for every cache format it supports and every split
plan; both must agree with the oracle."""
import numpy as np
import pytest
import torch

import paged_kv_cache_439_b200 as pkv
from paged_kv_cache_439_b200.workloads import make_custom, make_workload

from pkv_testlib import GpuCache, OracleCache, assert_close, bits, tol_for

pytestmark = pytest.mark.gpu


def _prefilled(wl):
    g = GpuCache(wl)
    g.append(wl.prefill_k, wl.prefill_v, wl.prefill_slots)
    return g


def _fused(g, wl, num_splits=0, slots=None):
    dev = g.device
    return pkv.paged_attention_decode_append(
        wl.q.to(dev), wl.new_k.to(dev), wl.new_v.to(dev),
        (wl.new_slots if slots is None else slots).to(dev), g.k, g.v,
        wl.block_tables.to(dev), wl.context_lens.to(dev), softmax_scale=wl.softmax_scale,
        k_scale=g.ks, v_scale=g.vs, max_context_len=wl.max_context_len, num_splits=num_splits,
        err_flag=g.err)


def _same_cache(a, b):
    assert np.array_equal(bits(a.k), bits(b.k))
    assert np.array_equal(bits(a.v), bits(b.v))
    if a.ks is not None:
        assert np.array_equal(bits(a.ks), bits(b.ks))
        assert np.array_equal(bits(a.vs), bits(b.vs))


@pytest.mark.parametrize("cache_dtype", ["bf16", "i8", "fp8"])
@pytest.mark.parametrize("group,d,bs", [(4, 128, 16), (1, 64, 16), (8, 128, 256), (16, 64, 8),
                                        (3, 128, 16), (12, 64, 16)])
def test_fused_step_equals_append_then_decode(cache_dtype, group, d, bs):
    lens = [1, 17, 100, 333, 64, 1024]
    wl = make_custom(f"fused-{cache_dtype}-{group}-{d}-{bs}", lens, 2 * group, 2, d, bs,
                     cache_dtype, seed=51)
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1, 3):
        two = _prefilled(wl)
        two.append(wl.new_k, wl.new_v, wl.new_slots)
        out_two = two.decode(num_splits=splits)
        one = _prefilled(wl)
        out_one = _fused(one, wl, num_splits=splits)
        torch.cuda.synchronize()
        assert one.flags() == 0 and two.flags() == 0
        _same_cache(one, two)
        assert np.array_equal(bits(out_one), bits(out_two)), f"splits={splits}"
        assert_close(out_one, ref, tol_for(wl), f"{wl.name} splits={splits}")


def test_mismatched_slot_writes_nothing_and_flags():
    wl = make_custom("fused-bad", [40, 70], 4, 2, 128, 16, "bf16", seed=52)
    g = _prefilled(wl)
    before_k, before_v = bits(g.k).copy(), bits(g.v).copy()
    slots = wl.new_slots.clone()
    slots[0] = slots[0] - 1          # a slot of the sequence, but not position ctx - 1
    slots[1] = -1                    # padding: nothing written, no flag
    _fused(g, wl, slots=slots)
    torch.cuda.synchronize()
    assert g.flags() & pkv.PKV_FLAG_BAD_SLOT
    assert np.array_equal(bits(g.k), before_k) and np.array_equal(bits(g.v), before_v)


def test_negative_slots_skip_the_append():
    wl = make_custom("fused-skip", [40, 70], 4, 2, 128, 16, "i8", seed=53)
    g = _prefilled(wl)
    before = bits(g.ks).copy()
    _fused(g, wl, slots=torch.full_like(wl.new_slots, -1))
    torch.cuda.synchronize()
    assert g.flags() == 0
    assert np.array_equal(bits(g.ks), before)


@pytest.mark.parametrize("name,kw", [("llama2-7b-mha", {}), ("llama2-13b-int8", {}),
                                     ("llama2-13b-int8", {"cache_dtype": "fp8"}),
                                     ("llama2-70b-gqa", {})])
def test_full_workloads_fused(name, kw):
    wl = make_workload(name, **kw)
    g = _prefilled(wl)
    out = _fused(g, wl)
    torch.cuda.synchronize()
    assert g.flags() == 0
    ref = OracleCache(wl).fill().decode()
    assert_close(out, ref, tol_for(wl), f"{name} fused")
