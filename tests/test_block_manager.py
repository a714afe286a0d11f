"""The host block manager (C++, through the C ABI): on-demand allocation at
block boundaries, ref counts, fork, copy-on-write of a shared partially filled
block, free on finish, swap bookkeeping, atomic failure.  No GPU needed."""
import random

import numpy as np
import pytest

from paged_kv_cache_439_b200 import _native as N
from paged_kv_cache_439_b200.block_manager import BlockManager


@pytest.fixture(autouse=True)
def _build():
    from paged_kv_cache_439_b200 import build
    build.build()


def test_allocation_on_demand_and_slots():
    m = BlockManager(8, 16)
    m.add_sequence(7)
    slots, cow = m.reserve(7, 40)
    assert cow is None
    # blocks come off the free list 0, 1, 2; slot = block * 16 + offset
    assert slots.tolist() == [b * 16 + o for b in range(3) for o in range(16)][:40]
    assert m.num_free == 5 and m.seq_len(7) == (40, 3)
    slots, _ = m.reserve(7, 9)      # 40..48: fills block 2, opens block 3 at token 48
    assert slots.tolist() == [2 * 16 + o for o in range(8, 16)] + [3 * 16]
    tables, lens = m.block_tables([7], 6)
    assert tables.tolist() == [[0, 1, 2, 3, -1, -1]] and lens.tolist() == [49]


def test_fork_copy_on_write_and_free():
    m = BlockManager(8, 16)
    m.add_sequence(1)
    m.reserve(1, 20)                # blocks 0 (full) and 1 (4 tokens)
    m.fork(1, 2)
    assert m.ref_count(0) == 2 and m.ref_count(1) == 2
    assert m.blocks_needed(2, 1) == 1
    slots, cow = m.reserve(2, 1)    # shared partial block 1 -> private copy
    assert cow == (1, 2)
    assert slots.tolist() == [2 * 16 + 4]
    assert m.ref_count(1) == 1 and m.ref_count(2) == 1 and m.ref_count(0) == 2
    t, l = m.block_tables([1, 2], 2)
    assert t.tolist() == [[0, 1], [0, 2]] and l.tolist() == [20, 21]
    # the parent's own next token needs no copy any more
    assert m.reserve(1, 1)[1] is None
    m.free(1)
    assert m.ref_count(0) == 1 and m.ref_count(1) == 0
    m.free(2)
    assert m.num_free == 8
    # freed blocks are reused last-in first-out: sequence 2 released 0, then 2
    m.add_sequence(3)
    assert m.reserve(3, 1)[0].tolist() == [2 * 16]


def test_fork_at_block_boundary_needs_no_copy():
    m = BlockManager(4, 16)
    m.add_sequence(1)
    m.reserve(1, 32)
    m.fork(1, 2)
    slots, cow = m.reserve(2, 1)
    assert cow is None and slots.tolist() == [2 * 16]


def test_exhaustion_is_atomic():
    m = BlockManager(3, 8)
    m.add_sequence(1)
    m.reserve(1, 20)                # 3 blocks
    with pytest.raises(N.PkvError) as e:
        m.reserve(1, 5)
    assert e.value.status == N.PKV_ERR_NO_BLOCKS
    assert m.seq_len(1) == (20, 3) and m.num_free == 0
    with pytest.raises(N.PkvError):
        m.fork(9, 10)               # unknown parent
    with pytest.raises(N.PkvError):
        m.block_tables([1], 2)      # table too narrow


def test_swap_out_and_in():
    dev = BlockManager(6, 16)
    host = BlockManager(10, 16)
    dev.add_sequence(5)
    dev.reserve(5, 40)
    out_pairs = dev.swap_out(host, 5)
    assert out_pairs[:, 0].tolist() == [0, 1, 2] and len(set(out_pairs[:, 1])) == 3
    assert dev.num_free == 6 and host.num_free == 7 and host.seq_len(5) == (40, 3)
    with pytest.raises(N.PkvError):
        dev.seq_len(5)
    in_pairs = host.swap_in(dev, 5)
    assert in_pairs[:, 0].tolist() == out_pairs[:, 1].tolist()
    assert dev.seq_len(5) == (40, 3) and host.num_free == 10
    # a shared block stays with the other sequence; the swapped one gets copies
    dev.fork(5, 6)
    pairs = dev.swap_out(host, 6)
    assert len(pairs) == 3 and all(dev.ref_count(b) == 1 for b in pairs[:, 0])


def test_random_operations_match_a_reference_model():
    rng = random.Random(4)
    NB, BS = 40, 8
    m = BlockManager(NB, BS)
    ref = {}          # seq -> (blocks, len)
    refcnt = [0] * NB
    free = list(range(NB - 1, -1, -1))
    nxt = 0
    for step in range(3000):
        op = rng.random()
        if op < 0.15 or not ref:
            m.add_sequence(nxt)
            ref[nxt] = ([], 0)
            nxt += 1
        elif op < 0.25:
            p = rng.choice(list(ref))
            m.fork(p, nxt)
            blocks, ln = ref[p]
            for b in blocks:
                refcnt[b] += 1
            ref[nxt] = (list(blocks), ln)
            nxt += 1
        elif op < 0.45:
            s = rng.choice(list(ref))
            m.free(s)
            for b in ref.pop(s)[0]:
                refcnt[b] -= 1
                if refcnt[b] == 0:
                    free.append(b)
        else:
            s = rng.choice(list(ref))
            n = rng.randint(1, 12)
            blocks, ln = ref[s]
            need = max(0, -(-(ln + n - len(blocks) * BS) // BS))
            cow = ln % BS != 0 and blocks and refcnt[blocks[-1]] > 1
            if need + cow > len(free):
                with pytest.raises(N.PkvError):
                    m.reserve(s, n)
                continue
            slots, pair = m.reserve(s, n)
            blocks = list(blocks)
            if cow:
                old = blocks[-1]
                new = free.pop()
                refcnt[new] = 1
                refcnt[old] -= 1
                if refcnt[old] == 0:
                    free.append(old)
                blocks[-1] = new
                assert pair == (old, new)
            else:
                assert pair is None
            expect = []
            for _ in range(n):
                if ln == len(blocks) * BS:
                    b = free.pop()
                    refcnt[b] = 1
                    blocks.append(b)
                expect.append(blocks[-1] * BS + ln % BS)
                ln += 1
            assert slots.tolist() == expect
            ref[s] = (blocks, ln)
        assert m.num_free == len(free)
    for b in range(NB):
        assert m.ref_count(b) == refcnt[b]
