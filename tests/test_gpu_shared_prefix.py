"""Shared-prefix (cascade) decode against the oracle and the plain decode.

Sequences of a batch share their first ``prefix_len`` tokens through the same
physical blocks (prefix caching).  The cascade call must give the attention
of the definition (checked against the oracle), whatever the group size,
head_dim, block size, row count or prefix/suffix split."""
import numpy as np
import pytest
import torch

import paged_kv_cache_439_b200 as pkv
from paged_kv_cache_439_b200.workloads import make_custom, make_workload

from pkv_testlib import GpuCache, OracleCache, assert_close, bits, tol_for

pytestmark = pytest.mark.gpu


def _cascade(g, wl, prefix_len, context_lens=None, **kw):
    dev = g.device
    cl = (wl.context_lens if context_lens is None else context_lens).to(dev)
    return pkv.paged_attention_decode_shared_prefix(
        wl.q.to(dev), g.k, g.v, wl.block_tables.to(dev), cl, prefix_len,
        softmax_scale=wl.softmax_scale, max_context_len=int(cl.max()), err_flag=g.err, **kw)


@pytest.mark.parametrize("group,d,bs", [(4, 128, 16), (1, 128, 16), (8, 128, 16), (16, 64, 16),
                                        (4, 64, 8), (8, 128, 256), (2, 128, 32), (3, 128, 16),
                                        (12, 64, 16)])
def test_shared_prefix_matches_oracle(group, d, bs):
    prefix = 256 if bs == 256 else 4 * bs * 8
    lens = [prefix + x for x in (1, 17, 100, 5, 64, 300)]
    wl = make_custom(f"sp-{group}-{d}-{bs}", lens, 2 * group, 2, d, bs, "bf16", seed=31,
                     shared_prefix=prefix)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1, 3):
        out = _cascade(g, wl, prefix, num_splits=splits)
        assert_close(out, ref, tol_for(wl), f"{wl.name} splits={splits}")
    assert g.flags() == 0
    # and it agrees with the plain decode of the same cache
    plain = g.decode()
    np.testing.assert_allclose(_cascade(g, wl, prefix).float().cpu().numpy(),
                               plain.float().cpu().numpy(), rtol=2e-2, atol=4e-3)


def test_many_rows_span_several_row_groups():
    # 40 sequences x group 8 = 320 q rows per KV head (several CTAs of rows)
    lens = [128 + 1 + (7 * i) % 90 for i in range(40)]
    wl = make_custom("sp-rows", lens, 16, 2, 128, 16, "bf16", seed=32, shared_prefix=128)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    assert_close(_cascade(g, wl, 128), ref, tol_for(wl), "rows")


def test_sequences_shorter_than_the_prefix():
    wl = make_custom("sp-short", [200, 150, 300], 8, 2, 128, 16, "bf16", seed=33, shared_prefix=128)
    g = GpuCache(wl).fill()
    cl = torch.tensor([200, 40, 0], dtype=torch.int32)   # 40 < prefix, 0 = empty
    out = _cascade(g, wl, 128, context_lens=cl)
    ref = OracleCache(wl).fill()
    wl.context_lens = cl
    r = ref.decode()
    assert_close(out, r, tol_for(wl), "short")
    assert (out[2] == 0).all()


def test_prefix_only_and_bad_prefix_block():
    wl = make_custom("sp-edge", [129, 130], 4, 1, 128, 16, "bf16", seed=34, shared_prefix=128)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    assert_close(_cascade(g, wl, 128), ref, tol_for(wl), "edge")
    bt = wl.block_tables.clone()
    bt[0, 2] = wl.num_blocks + 5                  # a bad entry inside the shared prefix
    out = pkv.paged_attention_decode_shared_prefix(
        wl.q.cuda(), g.k, g.v, bt.cuda(), wl.context_lens.cuda(), 128,
        softmax_scale=wl.softmax_scale, max_context_len=130, err_flag=g.err)
    torch.cuda.synchronize()
    assert g.flags() & 1
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("bs", [16, 256])
def test_full_shared_prefix_workload(bs):
    wl = make_workload("shared-prefix", block_size=bs)
    g = GpuCache(wl).fill()
    out = _cascade(g, wl, 4096)
    torch.cuda.synchronize()
    ref = OracleCache(wl).fill().decode()
    r = assert_close(out, ref, tol_for(wl), f"shared-prefix bs={bs}")
    assert g.flags() == 0
    print(f"shared-prefix cascade bs={bs}: max_abs={r['max_abs']:.2e}")


def test_ragged_prefix_tiles():
    # prefix of 40 tokens (5 blocks of 8): the shared slice ends inside a tile
    lens = [40 + x for x in (1, 9, 33, 70)]
    wl = make_custom("sp-ragged", lens, 8, 2, 128, 8, "bf16", seed=35, shared_prefix=40)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 2):
        assert_close(_cascade(g, wl, 40, num_splits=splits), ref, tol_for(wl), "ragged")
    assert g.flags() == 0


def test_running_max_moves_inside_the_prefix():
    """Keys of two later prefix blocks are scaled up so that, for many rows, a
    later tile's scores exceed everything before by far more than 2^8 in the
    exponent: the kernel must move its reference maximum and rescale O."""
    prefix, bs = 512, 16
    lens = [prefix + x for x in (3, 40, 77, 120, 1, 64, 200, 9)]
    wl = make_custom("sp-move", lens, 16, 2, 128, bs, "bf16", seed=36, shared_prefix=prefix)
    prefix_blocks = wl.block_tables[0, :prefix // bs]
    blk = wl.prefill_slots // bs
    for which, factor in ((5, 6.0), (20, 12.0)):   # tiles 1 and 5 of the prefix
        rows = (blk == prefix_blocks[which]).nonzero().flatten()
        wl.prefill_k[rows] = (wl.prefill_k[rows].float() * factor).to(wl.prefill_k.dtype)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1):
        assert_close(_cascade(g, wl, prefix, num_splits=splits), ref, tol_for(wl), "moving max")
    assert g.flags() == 0


@pytest.mark.parametrize("bs,moving", [(16, False), (256, False), (16, True)])
def test_prefix_slices_of_several_tiles(bs, moving):
    """64 KV heads of group 1 leave few prefix slices, each of several 64-token
    tiles: both score buffers take turns, S of tile j + 2 is computed behind
    P V of tile j, and (keys scaled up in two later tiles of the first slice)
    O is rescaled inside a slice."""
    prefix = 2048
    lens = [prefix + x for x in (1, 30, 77, 5, 160, 64, 9, 250)]
    wl = make_custom(f"sp-tiles-{bs}-{int(moving)}", lens, 64, 64, 128, bs, "bf16", seed=39,
                     shared_prefix=prefix)
    ps, _ = pkv.shared_prefix_plan(wl.num_seqs, 64, 64, 128, wl.max_context_len, prefix,
                                   torch.bfloat16, 0)
    assert 2 * 64 * ps <= prefix   # two tiles per slice at least
    if moving:
        prefix_blocks = wl.block_tables[0, :prefix // bs]
        blk = wl.prefill_slots // bs
        for which, factor in ((9, 6.0), (21, 12.0)):   # tiles 2 and 5 of the first slice
            rows = (blk == prefix_blocks[which]).nonzero().flatten()
            wl.prefill_k[rows] = (wl.prefill_k[rows].float() * factor).to(wl.prefill_k.dtype)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1):
        assert_close(_cascade(g, wl, prefix, num_splits=splits), ref, tol_for(wl), wl.name)
    assert g.flags() == 0


def test_repeated_calls_never_stall():
    """Many back-to-back calls, all split choices: the pipeline's hand-offs must
    never deadlock (a stalled CTA gives up after 2 s and sets PKV_FLAG_TIMEOUT)."""
    wl = make_workload("shared-prefix")
    g = GpuCache(wl).fill()
    q, bt, cl = wl.q.cuda(), wl.block_tables.cuda(), wl.context_lens.cuda()
    for it in range(60):
        pkv.paged_attention_decode_shared_prefix(
            q, g.k, g.v, bt, cl, 4096, softmax_scale=wl.softmax_scale,
            max_context_len=wl.max_context_len, num_splits=it % 3, err_flag=g.err)
    torch.cuda.synchronize()
    assert g.flags() == 0


def _cascade_append(g, wl, prefix_len, slots=None, **kw):
    dev = g.device
    return pkv.paged_attention_decode_shared_prefix_append(
        wl.q.to(dev), wl.new_k.to(dev), wl.new_v.to(dev),
        (wl.new_slots if slots is None else slots).to(dev), g.k, g.v,
        wl.block_tables.to(dev), wl.context_lens.to(dev), prefix_len,
        softmax_scale=wl.softmax_scale, max_context_len=int(wl.context_lens.max()),
        err_flag=g.err, **kw)


@pytest.mark.parametrize("bs", [16, 256])
def test_cascade_with_fused_append_equals_two_calls(bs):
    prefix = 256 if bs == 256 else 512
    lens = [prefix + x for x in (1, 17, 100, 5, 64, 300)]
    wl = make_custom(f"sp-fused-{bs}", lens, 8, 2, 128, bs, "bf16", seed=37, shared_prefix=prefix)
    ref = OracleCache(wl).fill().decode()
    for splits in (0, 1, 3):
        two = GpuCache(wl)
        two.append(wl.prefill_k, wl.prefill_v, wl.prefill_slots)
        two.append(wl.new_k, wl.new_v, wl.new_slots)
        out_two = _cascade(two, wl, prefix, num_splits=splits)
        one = GpuCache(wl)
        one.append(wl.prefill_k, wl.prefill_v, wl.prefill_slots)
        out_one = _cascade_append(one, wl, prefix, num_splits=splits)
        torch.cuda.synchronize()
        assert one.flags() == 0 and two.flags() == 0
        assert np.array_equal(bits(one.k), bits(two.k)) and np.array_equal(bits(one.v), bits(two.v))
        assert np.array_equal(bits(out_one), bits(out_two)), f"splits={splits}"
        assert_close(out_one, ref, tol_for(wl), f"{wl.name} splits={splits}")


def test_cascade_append_refuses_a_token_inside_the_shared_prefix():
    wl = make_custom("sp-fused-in", [200, 150], 4, 1, 128, 16, "bf16", seed=38, shared_prefix=128)
    g = GpuCache(wl)
    g.append(wl.prefill_k, wl.prefill_v, wl.prefill_slots)
    before = bits(g.k).copy()
    cl = torch.tensor([100, 150], dtype=torch.int32)   # sequence 0's position 99 is shared
    slots = wl.new_slots.clone()
    slots[1] = -1
    dev = g.device
    pkv.paged_attention_decode_shared_prefix_append(
        wl.q.to(dev), wl.new_k.to(dev), wl.new_v.to(dev), slots.to(dev), g.k, g.v,
        wl.block_tables.to(dev), cl.to(dev), 128, softmax_scale=wl.softmax_scale,
        max_context_len=150, err_flag=g.err)
    torch.cuda.synchronize()
    assert g.flags() & pkv.PKV_FLAG_BAD_SLOT
    assert np.array_equal(bits(g.k), before)


def test_full_shared_prefix_workload_fused_append():
    wl = make_workload("shared-prefix")
    g = GpuCache(wl)
    g.append(wl.prefill_k, wl.prefill_v, wl.prefill_slots)
    out = _cascade_append(g, wl, 4096)
    torch.cuda.synchronize()
    assert g.flags() == 0
    assert_close(out, OracleCache(wl).fill().decode(), tol_for(wl), "shared-prefix fused")
