"""Pins for the CPU oracle: it is checked against facts the pages and the
mathematics fix, never against itself or the CUDA path.

Sources: "LLM推理显存优化KV Cache管理3大策略" (mlqm.cn) §1-§4;
"生产级 LLM 推理的 KV 缓存优化" (GPUYard) §2; "大模型推理加速实战：KV Cache内存
优化与PagedAttention分页管理方案" (yunthe.com), PagedAttention section.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from paged_kv_cache_439_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- KV size

def _kv_size_rows():
    rows = []
    with open(os.path.join(GOLDEN, "kv_size_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split("|")
            rows.append((tuple(int(v) for v in lhs.split()), rhs.strip()))
    return rows


@pytest.mark.parametrize("args,expected", _kv_size_rows())
def test_kv_size_matches_pages(args, expected):
    got = oracle.kv_cache_bytes(*args)
    kind, val = expected.split(":")
    if kind == "exact":
        assert got == int(val)
    elif kind == "over_gb":
        assert got > float(val) * 1e9
    elif kind == "approx_gb":
        assert round(got / 1e9, 1) == float(val)
    else:  # pragma: no cover
        raise AssertionError(kind)


def test_kv_size_mha_vs_gqa_ratio():
    # the page's MHA figure is the GQA one with 64 instead of 8 KV heads
    gqa = oracle.kv_cache_bytes(1, 32768, 80, 8, 128, 2)
    mha = oracle.kv_cache_bytes(1, 32768, 80, 64, 128, 2)
    assert mha == 8 * gqa == 85_899_345_920
    # mlqm.cn §1: batch 8 is eight times one request ("16.8GB" = 8 x 2.1GB)
    assert oracle.kv_cache_bytes(8, 4096, 32, 32, 128, 2) == 8 * oracle.kv_cache_bytes(
        1, 4096, 32, 32, 128, 2)


# ---------------------------------------------------------------- block table

def _block_table_example():
    tables = {}
    with open(os.path.join(GOLDEN, "block_table_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            tables[key] = [int(v) for v in vals]
    return tables


def test_block_table_example_gather():
    ex = _block_table_example()
    bs = ex.pop("block_size")[0]
    nb = 8
    # each cache row stores its own (block, offset) so the gather is readable
    cache = np.zeros((nb, bs, 1, 2), dtype=np.float32)
    for b in range(nb):
        for o in range(bs):
            cache[b, o, 0] = (b, o)
    for name, table in ex.items():
        ctx = len(table) * bs
        rows = oracle.gather(cache, np.array(table, dtype=np.int32), ctx)
        # logical token t of the sequence lives in block table[t // 16], row t % 16
        for t in range(ctx):
            assert tuple(rows[t, 0]) == (table[t // bs], t % bs), (name, t)
    # spot values read straight off the page's picture: A's token 16 is the first
    # row of physical block 3, B's token 40 is row 8 of physical block 5
    rows_a = oracle.gather(cache, np.array(ex["A"], dtype=np.int32), 48)
    rows_b = oracle.gather(cache, np.array(ex["B"], dtype=np.int32), 48)
    assert tuple(rows_a[16, 0]) == (3, 0)
    assert tuple(rows_b[40, 0]) == (5, 8)


def test_append_places_rows_per_example():
    ex = _block_table_example()
    bs = ex.pop("block_size")[0]
    cache = np.full((8, bs, 2, 4), -1, dtype=np.int16)
    for seq_id, (name, table) in enumerate(ex.items()):
        T = len(table) * bs
        x = np.zeros((T, 2, 4), dtype=np.int16)
        x[:, :, 0] = seq_id
        x[:, :, 1] = np.arange(T)[:, None]
        slots = np.array([table[t // bs] * bs + t % bs for t in range(T)], dtype=np.int64)
        oracle.append_rows(x, slots, cache)
    assert (cache[[4, 6], :, :, :] == -1).all()          # untouched blocks
    assert (cache[0, :, :, 0] == 0).all() and (cache[1, :, :, 0] == 1).all()
    assert cache[7, 5, 1, 1] == 32 + 5                    # A: block 7 holds tokens 32..47
    assert cache[2, 3, 0, 1] == 16 + 3                    # B: block 2 holds tokens 16..31


def test_append_negative_slot_skipped_and_bad_slot_rejected():
    cache = np.zeros((2, 4, 1, 2), dtype=np.float32)
    x = np.ones((3, 1, 2), dtype=np.float32)
    oracle.append_rows(x, np.array([-1, 5, -7]), cache)
    assert cache.sum() == 2 and (cache[1, 1] == 1).all()
    with pytest.raises(oracle.OracleError):
        oracle.append_rows(x, np.array([0, 8, 1]), cache)


# ---------------------------------------------------------------- quantiser

def test_quantize_absmax_maps_to_127():
    rng = np.random.default_rng(1)
    for _ in range(200):
        x = rng.standard_normal(128).astype(np.float32) * rng.uniform(0.01, 50)
        codes, s = oracle.quantize_row(x)
        i = int(np.argmax(np.abs(x)))
        assert codes[i] == (127 if x[i] > 0 else -127)
        assert codes.min() >= -127 and codes.max() <= 127


def test_quantize_error_within_half_step():
    rng = np.random.default_rng(2)
    for _ in range(200):
        x = rng.standard_normal(64).astype(np.float32)
        x[rng.random(64) < 0.05] *= 8
        codes, s = oracle.quantize_row(x)
        # |x*s - code| <= 1/2 plus the rounding of the fp32 product x*s
        err = np.abs(x.astype(np.float64) * float(s) - codes.astype(np.float64))
        assert err.max() <= 0.5 + 127 * 2.0 ** -24
        # dequantised error is half a step 1/s (same slack)
        deq = codes.astype(np.float64) / float(s)
        assert np.abs(deq - x).max() <= (0.5 + 127 * 2.0 ** -24) / float(s)


def test_quantize_ties_round_half_to_even():
    # absmax 127 gives scale exactly 1, so x*s is exactly x and the .5 cases are ties
    x = np.array([127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -1.5, 126.5], dtype=np.float32)
    codes, s = oracle.quantize_row(x)
    assert s == np.float32(1.0)
    assert codes.tolist() == [127, 2, 4, -2, 0, 0, 2, -2, 126]
    # absmax 63.5 gives scale exactly 2: 0.25 -> 0.5 -> 0, 0.75 -> 1.5 -> 2
    y = np.array([63.5, 0.25, 0.75, -0.25, 1.25], dtype=np.float32)
    codes, s = oracle.quantize_row(y)
    assert s == np.float32(2.0)
    assert codes.tolist() == [127, 0, 2, 0, 2]


def test_quantize_zero_row_and_scale_is_fp32_quotient():
    codes, s = oracle.quantize_row(np.zeros(16, dtype=np.float32))
    assert s == np.float32(1.0) and (codes == 0).all()
    x = np.array([3.0, -7.0, 0.1], dtype=np.float32)
    _, s = oracle.quantize_row(x)
    # scale is the correctly rounded fp32 quotient 127 / 7
    assert s == np.float32(np.float32(127.0) / np.float32(7.0))
    assert abs(float(s) - 127.0 / 7.0) <= 2.0 ** -24 * 127.0 / 7.0


def test_quantize_is_fp32_not_fp64():
    # values whose fp32 product x*s rounds onto an exact .5 tie (then half-even)
    # while the exact product lies on the other side of the tie, so rounding the
    # unrounded (fp64) product would give the other integer
    absmax = np.float32(3.0)
    s32 = np.float32(127.0) / absmax
    cases = []
    for k in range(0, 126):
        target = np.float32(k + 0.5)
        x = np.float32(target / s32)
        for cand in (x, np.nextafter(x, np.float32(0)), np.nextafter(x, np.float32(100))):
            p32 = np.float32(cand * s32)
            p64 = float(cand) * float(s32)
            if p32 == target and round(p64) != int(np.rint(p32)):
                cases.append((cand, int(np.rint(p32))))
    assert len(cases) >= 5
    for cand, expect in cases:
        codes, s = oracle.quantize_row(np.array([absmax, cand], dtype=np.float32))
        assert s == s32
        assert codes[1] == expect, (cand, expect, codes[1])


def test_append_int8_layout():
    nb, bs, nkv, d = 3, 4, 2, 8
    codes = np.zeros((nb, bs, nkv, d), dtype=np.int8)
    scale = np.full((nb, nkv, bs), np.nan, dtype=np.float32)
    x = np.arange(2 * nkv * d, dtype=np.float32).reshape(2, nkv, d) - 10
    oracle.append_int8(x, np.array([5, -1 + 0 * 9], dtype=np.int64), codes, scale)
    # slot 5 = block 1, row 1; each head quantised on its own
    for h in range(nkv):
        c, s = oracle.quantize_row(x[0, h])
        assert (codes[1, 1, h] == c).all() and scale[1, h, 1] == s
    assert np.isnan(scale[0]).all() and np.isnan(scale[2]).all()
    assert np.isnan(scale[1, :, [0, 2, 3]]).all()


# ---------------------------------------------------------------- attention

def _random_paged(rng, lens, nq, nkv, d, bs, extra=3):
    need = sum((c + bs - 1) // bs for c in lens)
    nb = need + extra
    perm = rng.permutation(nb)
    k = rng.standard_normal((nb, bs, nkv, d)).astype(np.float32)
    v = rng.standard_normal((nb, bs, nkv, d)).astype(np.float32)
    maxb = max((c + bs - 1) // bs for c in lens) if lens else 1
    tables = np.full((len(lens), max(maxb, 1)), -1, dtype=np.int32)
    i = 0
    for s, c in enumerate(lens):
        for j in range((c + bs - 1) // bs):
            tables[s, j] = perm[i]
            i += 1
    q = rng.standard_normal((len(lens), nq, d)).astype(np.float32)
    return q, k, v, tables, np.array(lens, dtype=np.int32)


def _contiguous(cache, table, ctx, bs):
    return np.stack([cache[table[t // bs], t % bs] for t in range(ctx)]) if ctx else \
        np.zeros((0,) + cache.shape[2:], cache.dtype)


def _sdpa_reference(q, k, v, tables, lens, scale, bs):
    """torch's scaled_dot_product_attention in fp64 on contiguous K/V."""
    B, nq, d = q.shape
    nkv = k.shape[2]
    g = nq // nkv
    out = np.zeros((B, nq, d))
    for s in range(B):
        ctx = int(lens[s])
        if ctx == 0:
            continue
        K = torch.from_numpy(_contiguous(k, tables[s], ctx, bs).astype(np.float64))
        V = torch.from_numpy(_contiguous(v, tables[s], ctx, bs).astype(np.float64))
        K = K.permute(1, 0, 2).repeat_interleave(g, dim=0)  # [nq, ctx, d]
        V = V.permute(1, 0, 2).repeat_interleave(g, dim=0)
        Q = torch.from_numpy(q[s].astype(np.float64))[:, None, :]
        o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)
        out[s] = o[:, 0, :].numpy()
    return out


@pytest.mark.parametrize("nq,nkv,d,bs", [(4, 2, 64, 16), (8, 8, 32, 8), (8, 1, 16, 4),
                                         (16, 2, 128, 16)])
def test_paged_matches_library_sdpa(nq, nkv, d, bs):
    rng = np.random.default_rng(nq * 100 + nkv * 10 + bs)
    lens = [1, 5, bs, bs + 1, 3 * bs - 1, 70]
    q, k, v, tables, cl = _random_paged(rng, lens, nq, nkv, d, bs)
    scale = 1.0 / math.sqrt(d)
    got = oracle.paged_decode(q, k, v, tables, cl, scale)
    ref = _sdpa_reference(q, k, v, tables, cl, scale, bs)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_block_permutation_invariance_exact():
    rng = np.random.default_rng(7)
    bs = 16
    lens = [17, 33, 64, 100]
    q, k, v, tables, cl = _random_paged(rng, lens, 4, 2, 64, bs, extra=10)
    base = oracle.paged_decode(q, k, v, tables, cl, 0.125)
    nb = k.shape[0]
    perm = rng.permutation(nb)             # new position of each physical block
    k2 = np.empty_like(k)
    v2 = np.empty_like(v)
    k2[perm] = k
    v2[perm] = v
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
    moved = oracle.paged_decode(q, k2, v2, t2, cl, 0.125)
    assert np.array_equal(base, moved)


def test_all_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(3)
    bs, nkv, d = 8, 2, 16
    q, k, v, tables, cl = _random_paged(rng, [1, 7, 8, 29], 4, nkv, d, bs)
    k[:] = rng.standard_normal((1, 1, nkv, d)).astype(np.float32)  # same key at every slot
    got = oracle.paged_decode(q, k, v, tables, cl, 0.3)
    for s, ctx in enumerate(cl):
        V = _contiguous(v, tables[s], ctx, bs).astype(np.float64)
        for h in range(4):
            np.testing.assert_allclose(got[s, h], V[:, h // 2].mean(axis=0), rtol=0, atol=1e-13)


def test_zero_query_gives_mean_and_ctx1_gives_v():
    rng = np.random.default_rng(4)
    bs = 16
    q, k, v, tables, cl = _random_paged(rng, [1, 40], 2, 1, 32, bs)
    q[:] = 0
    got = oracle.paged_decode(q, k, v, tables, cl, 0.125)
    V0 = _contiguous(v, tables[0], 1, bs)
    assert np.array_equal(got[0, 0], V0[0, 0].astype(np.float64))      # ctx 1 -> that V row
    V1 = _contiguous(v, tables[1], 40, bs).astype(np.float64)
    np.testing.assert_allclose(got[1, 1], V1[:, 0].mean(axis=0), rtol=0, atol=1e-13)


def test_empty_context_gives_zero():
    rng = np.random.default_rng(5)
    q, k, v, tables, cl = _random_paged(rng, [0, 3], 2, 2, 8, 4)
    got = oracle.paged_decode(q, k, v, tables, cl, 1.0)
    assert (got[0] == 0).all() and np.abs(got[1]).sum() > 0


def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(6)
    bs, g = 16, 4
    q, k, v, tables, cl = _random_paged(rng, [5, 33, 48], 8, 2, 32, bs)
    gqa = oracle.paged_decode(q, k, v, tables, cl, 0.2)
    k_rep = np.repeat(k, g, axis=2)   # kv head j serves q heads j*g .. j*g+g-1
    v_rep = np.repeat(v, g, axis=2)
    mha = oracle.paged_decode(q, k_rep, v_rep, tables, cl, 0.2)
    assert np.array_equal(gqa, mha)
    # MQA: one kv head serves all q heads
    q1, k1, v1, t1, c1 = _random_paged(rng, [9, 20], 6, 1, 16, 8)
    mqa = oracle.paged_decode(q1, k1, v1, t1, c1, 0.5)
    rep = oracle.paged_decode(q1, np.repeat(k1, 6, axis=2), np.repeat(v1, 6, axis=2), t1, c1, 0.5)
    assert np.array_equal(mqa, rep)


def test_brute_force_tiny():
    rng = np.random.default_rng(8)
    bs = 4
    q, k, v, tables, cl = _random_paged(rng, [1, 3, 4, 9, 0], 4, 2, 6, bs)
    got = oracle.paged_decode(q, k, v, tables, cl, 0.7)
    bf = brute.paged_decode(q.tolist(), k.tolist(), v.tolist(), tables.tolist(), cl.tolist(), 0.7)
    np.testing.assert_allclose(got, np.array(bf), rtol=0, atol=1e-13)


def test_bad_block_id_is_an_error():
    rng = np.random.default_rng(9)
    q, k, v, tables, cl = _random_paged(rng, [20], 2, 2, 8, 8)
    tables[0, 1] = k.shape[0] + 3
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(q, k, v, tables, cl, 1.0)


def test_int8_decode_equals_decode_on_dequantised_values():
    rng = np.random.default_rng(10)
    bs, nkv, d = 16, 2, 32
    lens = [3, 17, 40]
    q, kf, vf, tables, cl = _random_paged(rng, lens, 4, nkv, d, bs)
    nb = kf.shape[0]
    kc = np.zeros((nb, bs, nkv, d), np.int8)
    vc = np.zeros_like(kc)
    ks = np.ones((nb, nkv, bs), np.float32)
    vs = np.ones_like(ks)
    slots = np.arange(nb * bs, dtype=np.int64)
    oracle.append_int8(kf.reshape(-1, nkv, d), slots, kc, ks)
    oracle.append_int8(vf.reshape(-1, nkv, d), slots, vc, vs)
    got = oracle.paged_decode_i8(q, kc, vc, ks, vs, tables, cl, 0.25)
    # the same attention on code/scale values computed here in fp64
    kd = kc.astype(np.float64) / ks.transpose(0, 2, 1)[..., None].astype(np.float64)
    vd = vc.astype(np.float64) / vs.transpose(0, 2, 1)[..., None].astype(np.float64)
    ref = _sdpa_reference(q, kd, vd, tables, cl, 0.25, bs)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # and the quantised result stays near the unquantised one
    plain = oracle.paged_decode(q, kf, vf, tables, cl, 0.25)
    assert np.abs(got - plain).max() < 0.1


def test_workload_tiny_through_oracle_matches_sdpa():
    wl = workloads.make_workload("tiny")
    nb, bs, nkv, d = wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_dim
    kc = np.full((nb, bs, nkv, d), np.nan, np.float32)
    vc = np.full_like(kc, np.nan)
    oracle.append_rows(wl.prefill_k.numpy(), wl.prefill_slots.numpy(), kc)
    oracle.append_rows(wl.prefill_v.numpy(), wl.prefill_slots.numpy(), vc)
    oracle.append_rows(wl.new_k.numpy(), wl.new_slots.numpy(), kc)
    oracle.append_rows(wl.new_v.numpy(), wl.new_slots.numpy(), vc)
    tables = wl.block_tables.numpy()
    cl = wl.context_lens.numpy()
    got = oracle.paged_decode(wl.q.numpy(), kc, vc, tables, cl, wl.softmax_scale)
    ref = _sdpa_reference(wl.q.numpy(), kc, vc, tables, cl, wl.softmax_scale, bs)
    assert np.isfinite(got).all()           # NaN-poisoned slots were never read
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- FP8 (E4M3)

def _torch_e4m3_value(code):
    return float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])


def test_e4m3_decode_matches_library_for_all_codes():
    for code in range(256):
        ours = oracle.e4m3_decode(code)
        ref = _torch_e4m3_value(code)
        if math.isnan(ref):
            assert math.isnan(ours) and (code & 0x7F) == 0x7F
        else:
            assert ours == ref, (code, ours, ref)
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9


def test_e4m3_encode_matches_library_rounding():
    rng = np.random.default_rng(12)
    xs = np.concatenate([rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 0.01,
                         rng.standard_normal(2000) * 30]).astype(np.float32)
    # exact midpoints between neighbouring finite values (ties -> even mantissa)
    vals = sorted({oracle.e4m3_decode(c) for c in range(0x7F) if not math.isnan(oracle.e4m3_decode(c))})
    mids = np.array([(a + b) / 2 for a, b in zip(vals, vals[1:])], dtype=np.float32)
    xs = np.concatenate([xs, mids, -mids])
    xs = xs[np.abs(xs) <= 448]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    # +-0 encode as the same magnitude
    assert np.array_equal(ours & 0x7F, ref & 0x7F)
    nz = (ref & 0x7F) != 0
    assert np.array_equal(ours[nz], ref[nz])


def test_e4m3_saturates_and_quantize_fp8_rules():
    assert oracle.e4m3_encode(1e6) == 0x7E and oracle.e4m3_encode(-500.0) == 0xFE
    assert oracle.e4m3_encode(448.0001) == 0x7E
    rng = np.random.default_rng(13)
    for _ in range(100):
        x = rng.standard_normal(128).astype(np.float32)
        x[rng.random(128) < 0.02] *= 8
        codes, s = oracle.quantize_row_fp8(x)
        assert s == np.float32(np.float32(448.0) / np.float32(np.abs(x).max()))
        i = int(np.argmax(np.abs(x)))
        assert codes[i] == (0x7E if x[i] > 0 else 0xFE)          # absmax -> +-448
        dq = np.array([oracle.e4m3_decode(c) for c in codes]) / float(s)
        # half a quantum: 2^-4 relative for normals, 2^-10 absolute (scaled) below
        bound = np.maximum(np.abs(x.astype(np.float64)) * 2.0 ** -4, 2.0 ** -10 / float(s))
        assert (np.abs(dq - x) <= bound * (1 + 1e-6)).all()
    codes, s = oracle.quantize_row_fp8(np.zeros(8, np.float32))
    assert s == np.float32(1.0) and (codes == 0).all()


def test_fp8_decode_equals_attention_on_dequantised_values():
    rng = np.random.default_rng(14)
    bs, nkv, d = 16, 2, 32
    q, kf, vf, tables, cl = _random_paged(rng, [5, 17, 40], 4, nkv, d, bs)
    nb = kf.shape[0]
    kc = np.zeros((nb, bs, nkv, d), np.uint8)
    vc = np.zeros_like(kc)
    ks = np.ones((nb, nkv, bs), np.float32)
    vs = np.ones_like(ks)
    slots = np.arange(nb * bs, dtype=np.int64)
    oracle.append_fp8(kf.reshape(-1, nkv, d), slots, kc, ks)
    oracle.append_fp8(vf.reshape(-1, nkv, d), slots, vc, vs)
    got = oracle.paged_decode_fp8(q, kc, vc, ks, vs, tables, cl, 0.25)
    table = np.array([oracle.e4m3_decode(c) for c in range(256)])
    kd = table[kc] / ks.transpose(0, 2, 1)[..., None].astype(np.float64)
    vd = table[vc] / vs.transpose(0, 2, 1)[..., None].astype(np.float64)
    ref = _sdpa_reference(q, kd, vd, tables, cl, 0.25, bs)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    plain = oracle.paged_decode(q, kf, vf, tables, cl, 0.25)
    assert np.abs(got - plain).max() < 0.2


def test_copy_blocks_definition():
    src = np.arange(5 * 3 * 2, dtype=np.int16).reshape(5, 3, 2)
    dst = np.full((4, 3, 2), -1, dtype=np.int16)
    oracle.copy_blocks(dst, src, np.array([[4, 0], [1, 3]], dtype=np.int32))
    assert (dst[0] == src[4]).all() and (dst[3] == src[1]).all()
    assert (dst[1] == -1).all() and (dst[2] == -1).all()
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(dst, src, np.array([[5, 0]], dtype=np.int32))


def _torch_e4m3_codes(y32: np.ndarray) -> np.ndarray:
    """torch's float8_e4m3fn rounding (a library codec) of fp32 values, as bytes."""
    return torch.from_numpy(np.ascontiguousarray(y32, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def _fp32_tie_rows(rng, n_rows=24, d=128):
    """Rows whose fp32 product x*scale lands exactly on a midpoint between two
    E4M3 values while the exact (fp64) product does not: encoding the fp64
    product, or rounding it twice, gives another code on these elements."""
    mids = []
    vals = sorted({oracle.e4m3_decode(c) for c in range(0x7F)
                   if not math.isnan(oracle.e4m3_decode(c))})
    for a, b in zip(vals[1:-1], vals[2:]):
        mids.append((a + b) / 2)
    rows, found = [], 0
    while len(rows) < n_rows:
        absmax = np.float32(rng.uniform(0.5, 20.0))
        s = np.float32(np.float32(448.0) / absmax)
        x = rng.standard_normal(d).astype(np.float32) * (absmax / 4)
        x[0] = absmax
        x = np.clip(x, -absmax, absmax)
        hits = 0
        for i in range(1, d):
            m = float(rng.choice(mids)) * (1 if rng.random() < 0.5 else -1)
            c0 = np.float32(m / float(s))
            for c in (c0, np.nextafter(c0, np.float32(np.inf)), np.nextafter(c0, np.float32(-np.inf))):
                p32 = np.float32(c) * s
                if abs(float(c)) <= float(absmax) and float(p32) == m and float(c) * float(s) != m:
                    x[i] = c
                    hits += 1
                    break
        if hits:
            found += hits
            rows.append(x)
    return np.stack(rows), found


def test_quantize_fp8_codes_equal_library_rounding_of_fp32_products():
    """FP8 rule (reading of the serving pages' --kv-cache-dtype fp8 flag, with the
    mlqm page's §4 per-token scale rule carried over): codes are the E4M3
    rounding, to nearest even with saturation, of the fp32 products x*scale.
    The oracle's codes must equal torch's float8_e4m3fn conversion of exactly
    those products, bit for bit (sign of zero included)."""
    rng = np.random.default_rng(439)
    rows = [rng.standard_normal(128).astype(np.float32) for _ in range(200)]
    for _ in range(100):                       # 1% outliers x8, as in the 13B workload
        x = rng.standard_normal(128).astype(np.float32)
        x[rng.random(128) < 0.01] *= 8
        rows.append(x)
    for _ in range(50):                        # products in the subnormal range and -0
        x = (rng.standard_normal(128) * 1e-4).astype(np.float32)
        x[0] = np.float32(3.0)
        x[1] = np.float32(-1e-9)
        rows.append(x)
    ties, n_ties = _fp32_tie_rows(rng)
    assert n_ties >= 100                       # the constructed cases are really there
    rows.extend(list(ties))
    for x in rows:
        codes, s = oracle.quantize_row_fp8(x)
        assert s == np.float32(np.float32(448.0) / np.float32(np.abs(x).max()))
        prod32 = x * s                          # numpy fp32 multiply: correctly rounded
        assert np.array_equal(codes, _torch_e4m3_codes(prod32))
    # the tie rows separate the fp32 reading from the fp64 one: on some of their
    # elements the E4M3 value nearest the exact product is not the one chosen
    vals = np.array(sorted({oracle.e4m3_decode(c) for c in range(0x7F)
                            if not math.isnan(oracle.e4m3_decode(c))}))
    differ = 0
    for x in ties:
        codes, s = oracle.quantize_row_fp8(x)
        prod64 = x.astype(np.float64) * np.float64(s)
        for p, c in zip(prod64, codes):
            nearest = vals[np.argmin(np.abs(vals - abs(p)))]
            differ += nearest != abs(oracle.e4m3_decode(int(c)))
    assert differ >= 20
