"""Host logic: the block allocator and the seeded workload generator."""
import pytest
import torch

from paged_kv_cache_439_b200 import workloads
from paged_kv_cache_439_b200.workloads import BlockAllocator


def test_allocator_free_list_and_ref_counts():
    a = BlockAllocator(4, torch.Generator().manual_seed(0))
    got = [a.allocate() for _ in range(4)]
    assert sorted(got) == [0, 1, 2, 3] and a.num_free == 0
    with pytest.raises(MemoryError):
        a.allocate()
    a.share(got[0])
    assert a.ref_count[got[0]] == 2
    a.free(got[0])
    assert a.num_free == 0          # still referenced once
    a.free(got[0])
    assert a.num_free == 1
    with pytest.raises(ValueError):
        a.free(got[0])              # double free
    assert a.allocate() == got[0]   # reclaimed block is reused


def test_allocator_is_seeded():
    a = BlockAllocator(50, torch.Generator().manual_seed(5))
    b = BlockAllocator(50, torch.Generator().manual_seed(5))
    assert [a.allocate() for _ in range(50)] == [b.allocate() for _ in range(50)]


def test_tiny_workload_shape():
    wl = workloads.make_workload("tiny")
    assert wl.context_lens.tolist() == [17, 33, 64, 100]
    assert wl.num_blocks == 64 and wl.block_size == 16
    # pre-fill holds ctx-1 tokens per sequence; the step appends the last one
    assert wl.prefill_slots.numel() == sum(c - 1 for c in [17, 33, 64, 100])
    # each sequence's blocks are distinct and inside the pool
    used = [b for s in range(4) for b in wl.block_tables[s].tolist() if b >= 0]
    assert len(used) == len(set(used)) == 2 + 3 + 4 + 7
    assert all(0 <= b < 64 for b in used)
    # the first two sequences' new tokens open a new block (16 -> 17, 32 -> 33)
    for s, ctx in [(0, 17), (1, 33)]:
        slot = int(wl.new_slots[s])
        assert slot // 16 == int(wl.block_tables[s, (ctx - 1) // 16]) and slot % 16 == 0
    assert wl.kv_bytes() == 214 * 2 * 2 * 64 * 4
    # reproducible
    again = workloads.make_workload("tiny")
    assert torch.equal(again.q, wl.q) and torch.equal(again.block_tables, wl.block_tables)


def test_named_workload_sizes():
    wl = workloads.make_workload("llama2-7b-mha", batch=2)
    assert wl.num_kv_heads == 32 and wl.head_dim == 128 and wl.q.dtype == torch.bfloat16
    full = workloads.make_workload("llama2-7b-mha")
    assert full.kv_bytes() == 536_870_912
    assert full.num_blocks == 2458   # ceil(1.2 x 2048 needed blocks)
    # per-sequence data do not depend on the batch size
    assert torch.equal(wl.q[1], full.q[1])


def test_shared_prefix_blocks_are_shared():
    wl = workloads.make_custom("sp", [40, 50, 36], 4, 2, 16, 16, "bf16", seed=3, shared_prefix=32)
    t = wl.block_tables
    assert torch.equal(t[0, :2], t[1, :2]) and torch.equal(t[0, :2], t[2, :2])
    for b in t[0, :2].tolist():
        assert wl.allocator.ref_count[b] == 3
    # the prefix is pre-filled once, suffixes per sequence
    assert wl.prefill_slots.numel() == 32 + (40 - 33) + (50 - 33) + (36 - 33)


def test_int8_workload_has_outliers():
    wl = workloads.make_workload("llama2-13b-int8", batch=1)
    assert wl.cache_dtype == "i8"
    x = wl.prefill_k.float().abs()
    assert x.max() > 8.0   # the x8 outliers are present
