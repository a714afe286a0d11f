"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Append and INT8 quantisation are compared bit for bit; attention within the
stated tolerances: bf16 and INT8 caches |d| <= 2e-3 + 1e-2 |ref|, fp32 caches
|d| <= 1e-4 max(1, |ref|).  Every cache is NaN-poisoned before the appends,
so a read outside a sequence's tokens shows up as a non-finite output.
"""
import math

import numpy as np
import pytest
import torch

from paged_kv_cache_439_b200 import workloads
from paged_kv_cache_439_b200.workloads import make_custom, make_workload

from pkv_testlib import (GpuCache, OracleCache, assert_close, bits, compare, oracle_bits,
                         tol_for)

pytestmark = pytest.mark.gpu

RAGGED = [1, 2, 15, 16, 17, 31, 33, 100, 255, 257, 1000]


def _wl(cache_dtype, nq, nkv, d, bs, lens=RAGGED, seed=11, **kw):
    idt = kw.pop("input_dtype", torch.float32 if cache_dtype == "f32" else torch.bfloat16)
    return make_custom(f"{cache_dtype}-{nq}-{nkv}-{d}-{bs}", lens, nq, nkv, d, bs, cache_dtype,
                       seed=seed, input_dtype=idt, **kw)


# ---------------------------------------------------------------- append

@pytest.mark.parametrize("cache_dtype,d,bs", [("f32", 64, 16), ("bf16", 128, 16),
                                              ("bf16", 64, 8), ("i8", 128, 16), ("i8", 64, 256),
                                              ("fp8", 128, 16), ("fp8", 64, 8)])
def test_append_bit_exact(cache_dtype, d, bs):
    wl = _wl(cache_dtype, 8, 4, d, bs, lens=[1, 40, 300], outlier_prob=0.01)
    g = GpuCache(wl).fill()
    o = OracleCache(wl).fill()
    torch.cuda.synchronize()
    assert np.array_equal(bits(g.k), oracle_bits(wl, o.k))
    assert np.array_equal(bits(g.v), oracle_bits(wl, o.v))
    if cache_dtype in ("i8", "fp8"):
        assert np.array_equal(bits(g.ks), o.ks.view(np.int32))
        assert np.array_equal(bits(g.vs), o.vs.view(np.int32))
    assert g.flags() == 0


@pytest.mark.parametrize("kv", ["i8", "fp8"])
def test_append_int8_full_13b_bulk(kv):
    """Bulk fill of the Llama-2-13B-shaped workload (65,504 pre-fill tokens),
    INT8 and FP8 caches, bit for bit."""
    wl = make_workload("llama2-13b-int8", cache_dtype=kv)
    g = GpuCache(wl).fill()
    o = OracleCache(wl).fill()
    torch.cuda.synchronize()
    assert np.array_equal(bits(g.k), o.k) and np.array_equal(bits(g.v), o.v)
    assert np.array_equal(bits(g.ks), o.ks.view(np.int32))
    assert np.array_equal(bits(g.vs), o.vs.view(np.int32))


def test_append_int8_halfway_codes_round_to_even():
    """A row whose max is 127 has scale exactly 1, so its products are the
    inputs themselves: halfway values must round to the even code, and the
    extreme codes must be exact (closed form, no oracle)."""
    wl = _wl("i8", 4, 2, 128, 16, lens=[8])
    g = GpuCache(wl)
    vals = [127.0, 2.5, -3.5, 0.5, -0.5, 126.5, 1.5, -1.5, -127.0, 64.5, -64.5, 0.0]
    want = [127, 2, -4, 0, 0, 126, 2, -2, -127, 64, -64, 0]
    k = torch.zeros(1, 2, 128, dtype=torch.bfloat16)
    k[0, 0, :len(vals)] = torch.tensor(vals, dtype=torch.bfloat16)
    k[0, 1, :len(vals)] = -torch.tensor(vals, dtype=torch.bfloat16)
    slot = 5
    g.append(k, k, torch.tensor([slot], dtype=torch.int64))
    torch.cuda.synchronize()
    codes = g.k.cpu().view(torch.int8).numpy().reshape(-1, 2, 128)[slot]
    assert codes[0, :len(vals)].tolist() == want
    assert codes[1, :len(vals)].tolist() == [-w if w != 0 else 0 for w in want]
    assert (codes[:, len(vals):] == 0).all()
    scales = g.ks.cpu().numpy().reshape(-1, 2, 16)[slot // 16, :, slot % 16]
    assert scales.tolist() == [1.0, 1.0]
    assert g.flags() == 0


def test_append_skips_negative_and_flags_bad_slots():
    wl = _wl("bf16", 4, 2, 64, 16, lens=[20])
    g = GpuCache(wl)
    before = bits(g.k).copy()
    k = torch.ones(3, 2, 64, dtype=torch.bfloat16)
    slots = torch.tensor([-1, wl.num_blocks * 16 + 5, 3], dtype=torch.int64)
    g.append(k, k, slots)
    torch.cuda.synchronize()
    after = bits(g.k)
    changed = np.argwhere((after != before).any(axis=(2, 3)))
    assert changed.tolist() == [[0, 3]]          # only slot 3 written
    assert g.flags() & 2


# ---------------------------------------------------------------- decode: small

@pytest.mark.parametrize("splits", [0, 1, 3])
def test_tiny_workload(splits):
    wl = make_workload("tiny")
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    out = g.decode(num_splits=splits)
    assert out.dtype == torch.float32
    assert_close(out, ref, tol_for(wl), f"tiny splits={splits}")
    assert g.flags() == 0


GRID = [(dt, g, d) for dt in ("bf16", "i8", "fp8", "f32") for g in (1, 4, 8, 16)
        for d in (64, 128)]


@pytest.mark.parametrize("cache_dtype,group,d", GRID)
def test_decode_dtype_group_headdim(cache_dtype, group, d):
    nkv = 2
    wl = _wl(cache_dtype, nkv * group, nkv, d, 16,
             outlier_prob=0.01 if cache_dtype in ("i8", "fp8") else 0)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1, 5):
        out = g.decode(num_splits=splits)
        assert_close(out, ref, tol_for(wl), f"{wl.name} splits={splits}")
    assert g.flags() == 0


@pytest.mark.parametrize("cache_dtype", ["bf16", "i8", "fp8", "f32"])
@pytest.mark.parametrize("group", [2, 3, 6, 12])
def test_decode_groups_not_filling_the_head_tile(cache_dtype, group):
    """Groups that leave head columns of the mma n-tile (8 heads, or 16 with two
    tiles above 8) unused: those columns are masked and never written."""
    nkv = 3
    wl = _wl(cache_dtype, nkv * group, nkv, 128, 16, seed=12,
             outlier_prob=0.01 if cache_dtype in ("i8", "fp8") else 0)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1, 3):
        out = g.decode(num_splits=splits)
        assert_close(out, ref, tol_for(wl), f"{wl.name} splits={splits}")
    assert g.flags() == 0


@pytest.mark.parametrize("cache_dtype,bs", [("bf16", 8), ("bf16", 32), ("bf16", 256),
                                            ("i8", 8), ("i8", 256), ("fp8", 8), ("fp8", 256),
                                            ("f32", 128)])
def test_decode_block_sizes(cache_dtype, bs):
    wl = _wl(cache_dtype, 16, 2, 128, bs)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1, 4):
        assert_close(g.decode(num_splits=splits), ref, tol_for(wl), f"bs={bs} s={splits}")


def test_fp32_cache_bf16_query():
    wl = _wl("f32", 4, 2, 64, 16, input_dtype=torch.bfloat16)
    # the fp32 cache holds the bf16 values widened exactly; q stays bf16
    for name in ("prefill_k", "prefill_v", "new_k", "new_v"):
        setattr(wl, name, getattr(wl, name).float())
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    out = g.decode()
    assert out.dtype == torch.bfloat16
    assert_close(out, ref, (2e-3, 1e-2), "f32 cache, bf16 q")


def test_mqa_single_kv_head():
    wl = _wl("bf16", 8, 1, 128, 16)
    g = GpuCache(wl).fill()
    assert_close(g.decode(), OracleCache(wl).fill().decode(), tol_for(wl), "mqa")


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("cache_dtype", ["bf16", "i8", "fp8"])
def test_block_permutation_gives_bit_identical_output(cache_dtype):
    a = _wl(cache_dtype, 32, 4, 128, 16, placement_seed=1)
    b = _wl(cache_dtype, 32, 4, 128, 16, placement_seed=2)
    assert not torch.equal(a.block_tables, b.block_tables)
    ga = GpuCache(a).fill()
    gb = GpuCache(b).fill()
    for splits in (1, 3):
        assert np.array_equal(bits(ga.decode(num_splits=splits)),
                              bits(gb.decode(num_splits=splits)))


def test_deterministic_reruns():
    wl = _wl("bf16", 64, 8, 128, 16)
    g = GpuCache(wl).fill()
    a = bits(g.decode())
    for _ in range(3):
        assert np.array_equal(a, bits(g.decode()))


def test_splits_agree():
    wl = _wl("bf16", 16, 2, 128, 16, lens=[3000, 4097, 17])
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    outs = [g.decode(num_splits=s) for s in (1, 2, 7, 64)]
    for o in outs:
        assert_close(o, ref, tol_for(wl), "splits")


# ---------------------------------------------------------------- edges

@pytest.mark.parametrize("cache_dtype", ["bf16", "i8", "fp8"])
def test_empty_and_single_token_contexts(cache_dtype):
    wl = _wl(cache_dtype, 8, 2, 128, 16, lens=[0, 1, 0, 2, 16])
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1, 2):
        out = g.decode(num_splits=splits)
        assert (out[0] == 0).all() and (out[2] == 0).all()
        assert_close(out, ref, tol_for(wl), f"edges s={splits}")


@pytest.mark.parametrize("cache_dtype", ["bf16", "i8", "fp8"])
def test_padded_table_entries_never_read(cache_dtype):
    # entries past each sequence's last block point outside the pool
    wl = _wl(cache_dtype, 8, 2, 64, 16, lens=[5, 40], pad_entry=10**6, extra_table_cols=3)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode(block_tables=torch.where(
        wl.block_tables >= wl.num_blocks, torch.full_like(wl.block_tables, -1), wl.block_tables))
    assert_close(g.decode(), ref, tol_for(wl), "padded")
    assert g.flags() == 0


@pytest.mark.parametrize("cache_dtype", ["bf16", "i8", "fp8"])
def test_bad_block_sets_flag_and_is_skipped(cache_dtype):
    wl = _wl(cache_dtype, 8, 2, 64, 16, lens=[64, 40])
    g = GpuCache(wl).fill()
    bt = wl.block_tables.clone()
    bt[0, 1] = wl.num_blocks + 3          # tokens 16..31 of sequence 0 are unreachable
    out = g.decode(block_tables=bt)
    torch.cuda.synchronize()
    assert g.flags() & 1
    assert torch.isfinite(out.float()).all()
    # sequence 1 is untouched by the bad entry of sequence 0
    ref = OracleCache(wl).fill().decode()
    assert_close(out[1:], ref[1:], tol_for(wl), "other sequence")


def test_context_range_flags():
    wl = _wl("bf16", 8, 2, 64, 16, lens=[40, 20])
    g = GpuCache(wl).fill()
    g.decode(context_lens=torch.tensor([-3, 20], dtype=torch.int32))
    torch.cuda.synchronize()
    assert g.flags() & 8
    g.err.zero_()
    out = g.decode(context_lens=torch.tensor([40, 20], dtype=torch.int32), max_context_len=30)
    torch.cuda.synchronize()
    assert g.flags() & 4
    assert torch.isfinite(out.float()).all()


def test_error_status_from_binding():
    import paged_kv_cache_439_b200 as pkv
    wl = _wl("bf16", 8, 2, 64, 16, lens=[40])
    g = GpuCache(wl).fill()
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_attention_decode(wl.q.cuda(), g.k, g.v, wl.block_tables.cuda(),
                                   wl.context_lens.cuda(), workspace=ws, num_splits=3,
                                   max_context_len=40)
    assert e.value.status == -5


# ---------------------------------------------------------------- full-size workloads

FULL = [("llama2-7b-mha", None, None), ("llama2-70b-gqa", None, None),
        ("llama2-13b-int8", None, None), ("llama2-13b-int8", None, "fp8"),
        ("shared-prefix", 16, None), ("shared-prefix", 256, None)]


@pytest.mark.parametrize("name,bs,kv", FULL)
def test_full_workload_parity(name, bs, kv):
    """The workloads at full size, in the launch configuration the benchmark times."""
    wl = make_workload(name, block_size=bs, **({"cache_dtype": kv} if kv else {}))
    g = GpuCache(wl).fill()
    out = g.decode(num_splits=0)
    torch.cuda.synchronize()
    ref = OracleCache(wl).fill().decode()
    r = assert_close(out, ref, tol_for(wl), name)
    assert g.flags() == 0
    print(f"{name} bs={wl.block_size}: max_abs={r['max_abs']:.2e} max_rel={r['max_rel']:.2e}")


@pytest.mark.parametrize("cache_dtype", ["i8", "fp8", "bf16"])
def test_query_spread_over_many_binades(cache_dtype):
    """q elements spread over 24 binades (so they do not share one exponent):
    the one-byte engines' score paths stay within the stated tolerance."""
    wl = _wl(cache_dtype, 8, 8, 128, 16, lens=[33, 700, 2048], outlier_prob=0.01)
    gen = torch.Generator().manual_seed(5)
    mag = torch.pow(2.0, torch.randint(-20, 5, wl.q.shape, generator=gen).float())
    wl.q = (torch.randn(wl.q.shape, generator=gen) * mag).to(wl.q.dtype)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1, 3):
        assert_close(g.decode(num_splits=splits), ref, tol_for(wl), f"spread s={splits}")
