"""Pins for the block-manager oracle model against the rules and figures the pages print.

"PagedAttention原理": 从虚拟内存的启发 (one block of B at a time, waste < B), block_size 选取 (expected
waste (B-1)/2; sizes 8/16/32), 解决共享prompt / 解决COW (ref counts, the five COW steps), COW 区别
(append in place when there is room).  "Paged Attention&Orca Paper笔记与解读": parallel sampling and
beam search (blocks shared by forked sequences, freed at count 0).
"""
import copy
import json
import os

import pytest

from oracle.allocator import BlockManagerModel, NoFreeBlock, InvalidArg

FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")))
BLOCK_SIZES = FACTS["block_sizes"]["values"]


def _invariants(m: BlockManagerModel):
    used = sum(1 for r in m.ref if r > 0)
    assert used + m.num_free() == m.n_blocks
    assert len(set(m.free)) == len(m.free)
    assert all(m.ref[b] == 0 for b in m.free)
    # every reference comes from a sequence's block table
    refs = [0] * m.n_blocks
    for s in m.seqs.values():
        for b in s["table"]:
            refs[b] += 1
        assert len(s["table"]) == -(-s["n"] // m.B)
    assert refs == m.ref


@pytest.mark.parametrize("B", BLOCK_SIZES)
def test_blocks_allocated_on_demand_waste_below_B(B):
    m = BlockManagerModel(4096, B)
    for c in range(1, 5 * B + 2):
        sid = m.seq_create()
        slots, pairs = m.reserve_slots(sid, c)
        assert pairs == []
        nb = len(m.seq_table(sid))
        assert nb == -(-c // B)
        assert 0 <= nb * B - c <= B - 1          # internal waste bounded by one block
        # slot ids are block*B + offset in logical order
        t = m.seq_table(sid)
        assert slots == [t[i // B] * B + i % B for i in range(c)]
        m.seq_free(sid)
        _invariants(m)
    assert m.num_free() == 4096


@pytest.mark.parametrize("B", BLOCK_SIZES)
def test_expected_waste_is_half_block(B):
    # Over lengths spanning whole periods of B, the waste takes each value 0..B-1 equally often,
    # so its mean is exactly (B-1)/2 as printed.
    m = BlockManagerModel(100000, B)
    wastes = []
    for c in range(1, 8 * B + 1):
        sid = m.seq_create()
        m.reserve_slots(sid, c)
        wastes.append(len(m.seq_table(sid)) * B - c)
    assert sum(wastes) / len(wastes) == (B - 1) / 2
    assert FACTS["expected_internal_waste_tokens"]["formula"] == "(B-1)/2"


def test_one_token_at_a_time_equals_bulk():
    B = 16
    a, b = BlockManagerModel(64, B), BlockManagerModel(64, B)
    sa, sb = a.seq_create(), b.seq_create()
    slots_a = []
    for _ in range(77):
        s, p = a.reserve_slots(sa, 1)
        slots_a += s
        assert p == []
    slots_b, _ = b.reserve_slots(sb, 77)
    assert slots_a == slots_b and a.ref == b.ref and a.free == b.free


def test_fork_shares_blocks_and_counts_references():
    B = 8
    m = BlockManagerModel(32, B)
    p = m.seq_create()
    m.reserve_slots(p, 20)          # 3 blocks, last one partial (4 of 8)
    kids = [m.seq_fork(p) for _ in range(3)]
    for b in m.seq_table(p):
        assert m.refcount(b) == 4
    for k in kids:
        assert m.seq_table(k) == m.seq_table(p) and m.seq_len(k) == 20
    _invariants(m)


@pytest.mark.parametrize("N", [2, 3, 4])
def test_cow_on_shared_partial_block(N):
    # "解决COW": count 1 -> write in place; otherwise allocate, copy, remap, decrement, write.
    B = 16
    m = BlockManagerModel(128, B)
    p = m.seq_create()
    m.reserve_slots(p, 1024 + 7)       # prompt with a partial last block
    seqs = [p] + [m.seq_fork(p) for _ in range(N - 1)]
    tail = m.seq_table(p)[-1]
    full = m.seq_table(p)[:-1]
    assert m.refcount(tail) == N
    free0 = m.num_free()
    all_pairs = []
    for i, s in enumerate(seqs):
        before = m.refcount(tail)
        slots, pairs = m.reserve_slots(s, 1)
        if i < N - 1:
            assert len(pairs) == 1 and pairs[0][0] == tail          # steps 1-2
            new = pairs[0][1]
            assert m.seq_table(s)[-1] == new                          # step 3
            assert m.refcount(tail) == before - 1                     # step 4
            assert slots == [new * B + 7]                             # step 5
            assert m.refcount(new) == 1
        else:
            assert pairs == [] and slots == [tail * B + 7]            # last writer: in place
        all_pairs += pairs
    assert len(all_pairs) == N - 1 and m.num_free() == free0 - (N - 1)
    assert m.refcount(tail) == 1
    for b in full:                     # the full prompt blocks stay shared
        assert m.refcount(b) == N
    _invariants(m)


def test_full_shared_block_gets_fresh_block_without_copy():
    # "COW 区别": copying is only for writes into a block; a full last block is not written into.
    B = 16
    m = BlockManagerModel(16, B)
    p = m.seq_create()
    m.reserve_slots(p, 32)
    k = m.seq_fork(p)
    slots, pairs = m.reserve_slots(k, 1)
    assert pairs == [] and len(m.seq_table(k)) == 3 and m.seq_table(k)[:2] == m.seq_table(p)
    assert m.refcount(m.seq_table(k)[2]) == 1


def test_partial_unshared_block_is_appended_in_place():
    B = 16
    m = BlockManagerModel(16, B)
    p = m.seq_create()
    m.reserve_slots(p, 5)
    t = m.seq_table(p)
    slots, pairs = m.reserve_slots(p, 3)
    assert pairs == [] and m.seq_table(p) == t and slots == [t[0] * B + 5, t[0] * B + 6, t[0] * B + 7]


def test_free_at_zero_and_lifo_reuse():
    B = 8
    m = BlockManagerModel(8, B)
    a = m.seq_create()
    m.reserve_slots(a, 16)
    b = m.seq_fork(a)
    ta = m.seq_table(a)
    m.seq_free(a)
    assert all(m.refcount(x) == 1 for x in ta)    # still held by b
    m.seq_free(b)
    assert all(m.refcount(x) == 0 for x in ta)    # released at zero
    assert m.alloc_block() == ta[-1]              # most recently freed block comes back first
    assert m.num_free() == m.n_blocks - 1


def test_exhaustion_fails_and_changes_nothing():
    B = 16
    m = BlockManagerModel(5, B)
    p = m.seq_create()
    m.reserve_slots(p, 40)           # 3 blocks, partial
    k = m.seq_fork(p)
    snap = copy.deepcopy(m.__dict__)
    with pytest.raises(NoFreeBlock):
        m.reserve_slots(k, 1 + 3 * B)  # needs a COW block plus 3 fresh ones; only 2 free
    assert m.__dict__ == snap
    with pytest.raises(InvalidArg):
        m.decref(4)                   # not allocated


def test_beam_search_refcounts_stay_in_range():
    # Beam width k: a block's count is the number of live beams that descend through it.
    import random
    rnd = random.Random(0)
    B, k = 4, 4
    m = BlockManagerModel(4096, B)
    root = m.seq_create()
    m.reserve_slots(root, 9)
    beams = [root] + [m.seq_fork(root) for _ in range(k - 1)]
    for step in range(40):
        parents = [rnd.choice(beams) for _ in range(k)]
        new = [m.seq_fork(p) for p in parents]
        for b in beams:
            m.seq_free(b)
        beams = new
        for b in beams:
            m.reserve_slots(b, 1)
        _invariants(m)
        for b in set(x for s in beams for x in m.seq_table(s)):
            assert 1 <= m.refcount(b) <= k
    for b in beams:
        m.seq_free(b)
    assert m.num_free() == 4096


def test_block_tables_pack_and_pad():
    B = 8
    m = BlockManagerModel(32, B)
    a, b = m.seq_create(), m.seq_create()
    m.reserve_slots(a, 9)
    m.reserve_slots(b, 20)
    tables, lens = m.build_block_tables([b, a], 4)
    assert lens == [20, 9]
    assert tables[0][:3] == m.seq_table(b) and tables[0][3] == -1
    assert tables[1][:2] == m.seq_table(a) and tables[1][2:] == [-1, -1]
    with pytest.raises(InvalidArg):
        m.build_block_tables([b], 2)
