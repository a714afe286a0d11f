"""Block copies for copy-on-write and swap, driven by the host block manager,
checked bit for bit against the oracle's block copy and, end to end, by decode
parity against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_439_b200 as pkv
from paged_kv_cache_439_b200.block_manager import BlockManager, copy_blocks
from paged_kv_cache_439_b200.workloads import make_custom

from pkv_testlib import GpuCache, OracleCache, assert_close, bits, tol_for

pytestmark = pytest.mark.gpu


def _pairs(p):
    return torch.tensor(np.asarray(p, dtype=np.int32).reshape(-1, 2), device="cuda")


@pytest.mark.parametrize("cache_dtype", ["bf16", "i8", "fp8"])
def test_copy_blocks_device_to_device(cache_dtype):
    wl = make_custom("cp", [100, 60], 8, 2, 128, 16, cache_dtype, seed=41)
    g = GpuCache(wl).fill()
    o = OracleCache(wl).fill()
    s0, s1 = int(wl.block_tables[0, 0]), int(wl.block_tables[1, 2])
    d0, d1 = [b for b in range(wl.num_blocks) if b not in (s0, s1)][:2]
    pairs = np.array([[s0, d0], [s1, d1]], np.int32)
    copy_blocks(g.k, g.v, g.k, g.v, _pairs(pairs), g.ks, g.vs, g.ks, g.vs, err_flag=g.err)
    torch.cuda.synchronize()
    kref, vref = o.k.copy(), o.v.copy()
    oracle.copy_blocks(kref, o.k, pairs)
    oracle.copy_blocks(vref, o.v, pairs)
    assert np.array_equal(bits(g.k).reshape(kref.shape).view(kref.dtype), kref)
    assert np.array_equal(bits(g.v).reshape(vref.shape).view(vref.dtype), vref)
    if g.ks is not None:
        sref = o.ks.copy()
        oracle.copy_blocks(sref, o.ks, pairs)
        assert np.array_equal(bits(g.ks), sref.view(np.int32))
    assert g.flags() == 0


def test_copy_on_write_end_to_end():
    """Fork a sequence whose last block is partly full, let the child append:
    the block manager asks for a private copy, the kernel makes it, and both
    sequences then decode to the oracle's answers."""
    nkv, d, bs = 2, 128, 16
    m = BlockManager(16, bs)
    rng = torch.Generator().manual_seed(5)
    k_parent = torch.randn(20, nkv, d, generator=rng).to(torch.bfloat16)
    v_parent = torch.randn(20, nkv, d, generator=rng).to(torch.bfloat16)
    k_child = torch.randn(1, nkv, d, generator=rng).to(torch.bfloat16)
    v_child = torch.randn(1, nkv, d, generator=rng).to(torch.bfloat16)
    q = torch.randn(2, 8, d, generator=rng).to(torch.bfloat16)
    m.add_sequence(0)
    slots_p, _ = m.reserve(0, 20)
    m.fork(0, 1)
    slots_c, cow = m.reserve(1, 1)
    assert cow is not None
    kc = torch.full((16, bs, nkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp = torch.from_numpy(slots_p).cuda()
    pkv.kv_cache_append(k_parent.cuda(), v_parent.cuda(), sp, kc, vc, err_flag=err)
    copy_blocks(kc, vc, kc, vc, _pairs(cow), err_flag=err)
    pkv.kv_cache_append(k_child.cuda(), v_child.cuda(), torch.from_numpy(slots_c).cuda(), kc, vc,
                        err_flag=err)
    tables, lens = m.block_tables([0, 1], 2)
    out = pkv.paged_attention_decode(q.cuda(), kc, vc, torch.from_numpy(tables).cuda(),
                                     torch.from_numpy(lens).cuda(), max_context_len=21,
                                     err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # oracle: its own cache built from the same rows and slots, its own copy
    ko = np.full((16, bs, nkv, d), 0x7FC0, np.uint16)
    vo = ko.copy()
    rows = lambda x: x.view(torch.int16).numpy().view(np.uint16)
    oracle.append_rows(rows(k_parent), slots_p, ko)
    oracle.append_rows(rows(v_parent), slots_p, vo)
    oracle.copy_blocks(ko, ko.copy(), np.asarray(cow, np.int32).reshape(1, 2))
    oracle.copy_blocks(vo, vo.copy(), np.asarray(cow, np.int32).reshape(1, 2))
    oracle.append_rows(rows(k_child), slots_c, ko)
    oracle.append_rows(rows(v_child), slots_c, vo)
    widen = lambda b: (b.astype(np.uint32) << 16).view(np.float32)
    ref = oracle.paged_decode(q.float().numpy(), widen(ko), widen(vo), tables, lens,
                              1 / np.sqrt(d))
    assert_close(out, ref, (2e-3, 1e-2), "cow")
    # the parent never saw the child's token: its 20 tokens stay in the shared block
    assert tables[0, 1] == cow[0] and tables[1, 1] == cow[1]


def test_swap_round_trip_through_pinned_host_memory():
    wl = make_custom("swap", [300, 170, 33], 8, 2, 128, 16, "bf16", seed=42, pool_factor=2.0)
    g = GpuCache(wl).fill()
    ref = OracleCache(wl).fill().decode()
    nb = wl.num_blocks
    host_k = torch.empty((64,) + tuple(g.k.shape[1:]), dtype=g.k.dtype).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    # sequence 0 out to host blocks 10.., then back into fresh device blocks
    used = wl.block_tables[0][wl.block_tables[0] >= 0].tolist()
    out_pairs = np.array([[b, 10 + i] for i, b in enumerate(used)], np.int32)
    copy_blocks(host_k, host_v, g.k, g.v, _pairs(out_pairs), err_flag=g.err)
    torch.cuda.synchronize()
    assert np.array_equal(bits(host_k[10:10 + len(used)]), bits(g.k[used]))
    # the device blocks get reused (poisoned here), the sequence comes back elsewhere
    free = [b for b in range(nb) if b not in set(wl.block_tables.flatten().tolist())]
    assert len(free) >= len(used)
    g.k[used] = float("nan")
    g.v[used] = float("nan")
    back = np.array([[10 + i, free[i]] for i in range(len(used))], np.int32)
    copy_blocks(g.k, g.v, host_k, host_v, _pairs(back), err_flag=g.err)
    bt = wl.block_tables.clone()
    bt[0, :len(used)] = torch.tensor(free[:len(used)], dtype=torch.int32)
    out = g.decode(block_tables=bt)
    torch.cuda.synchronize()
    assert_close(out, ref, tol_for(wl), "after swap-in")
    assert g.flags() == 0


def test_bad_pairs_flag_and_skip():
    wl = make_custom("bad", [40], 4, 2, 64, 16, "bf16", seed=43)
    g = GpuCache(wl).fill()
    before = bits(g.k).copy()
    copy_blocks(g.k, g.v, g.k, g.v, _pairs([[wl.num_blocks + 2, 0]]), err_flag=g.err)
    torch.cuda.synchronize()
    assert g.flags() & pkv.PKV_FLAG_BAD_BLOCK
    assert np.array_equal(bits(g.k), before)


def test_probe_kernels_copy_and_read():
    """The two in-process HBM probes: pkv_copy moves every byte (ragged size,
    not a multiple of the grid), pkv_read XOR-folds every 16-byte vector."""
    import paged_kv_cache_439_b200 as pkv
    n = (3 << 20) + 16 * 37
    src = torch.randint(-2**31, 2**31 - 1, (n // 4,), dtype=torch.int32, device="cuda")
    dst = torch.zeros_like(src)
    pkv.copy(dst, src)
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.read(src, sink)
    pkv.read(src, sink)      # XOR twice: back to zero
    torch.cuda.synchronize()
    assert torch.equal(dst, src)
    assert int(sink.item()) == 0
    pkv.read(src, sink)
    words = src.cpu().numpy().view(np.uint32)
    expect = int(np.bitwise_xor.reduce(words))
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == expect
