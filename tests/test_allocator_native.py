"""The native block manager (pa_alloc_*, pa_seq_*) against the oracle model, bit for bit:
block ids, reference counts, free counts, slots, copy pairs and packed tables."""
import random

import pytest
import torch

from oracle.allocator import BlockManagerModel, NoFreeBlock as ModelNoFree, InvalidArg as ModelInvalid
from paged_kv_cache_329_b200 import api


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_329_b200 import build

    build.build()


def _same_state(nat: api.BlockManager, mod: BlockManagerModel):
    assert nat.num_free() == mod.num_free()
    for b in range(mod.n_blocks):
        assert nat.refcount(b) == mod.refcount(b)
    for sid in mod.seqs:
        assert nat.seq_len(sid) == mod.seq_len(sid)
        assert nat.seq_num_blocks(sid) == len(mod.seq_table(sid))


def _run_script(B, n_blocks, seed, steps=400):
    rnd = random.Random(seed)
    nat, mod = api.BlockManager(n_blocks, B), BlockManagerModel(n_blocks, B)
    live = []
    for _ in range(steps):
        op = rnd.random()
        if op < 0.15 or not live:
            a, b = nat.seq_create(), mod.seq_create()
            assert a == b
            live.append(a)
        elif op < 0.3:
            p = rnd.choice(live)
            a, b = nat.seq_fork(p), mod.seq_fork(p)
            assert a == b
            live.append(a)
        elif op < 0.4 and len(live) > 1:
            s = live.pop(rnd.randrange(len(live)))
            nat.seq_free(s)
            mod.seq_free(s)
        else:
            s = rnd.choice(live)
            n = rnd.choice([1, 1, 1, 2, 3, B - 1, B, B + 1, 3 * B])
            try:
                ref = mod.reserve_slots(s, n)
            except ModelNoFree:
                with pytest.raises(api.NoFreeBlock):
                    nat.reserve_slots(s, n)
            else:
                got = nat.reserve_slots(s, n)
                assert got[0] == ref[0] and [tuple(p) for p in got[1]] == [tuple(p) for p in ref[1]]
        _same_state(nat, mod)
    if live:
        mb = max(len(mod.seq_table(s)) for s in live) + 2
        t_nat, l_nat = nat.build_block_tables(live, mb)
        t_mod, l_mod = mod.build_block_tables(live, mb)
        assert t_nat.tolist() == t_mod and l_nat.tolist() == l_mod
    return nat, mod


@pytest.mark.parametrize("B", [8, 16, 32])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_scripts_match_model(B, seed):
    _run_script(B, 64 if seed != 2 else 12, seed)   # seed 2: a tight pool that runs out


def test_shared_prefix_trajectory_matches_model():
    # 32 requests x 4 sequences share a 1024-token prompt; each step every sequence picks a parent
    # among its request's 4 (beam-style fork), then reserves one slot.
    B, reqs, width = 16, 4, 4
    nat, mod = api.BlockManager(2048, B), BlockManagerModel(2048, B)
    rnd = random.Random(7)
    groups = []
    for r in range(reqs):
        root_n, root_m = nat.seq_create(), mod.seq_create()
        assert root_n == root_m
        nat.reserve_slots(root_n, 1024)
        mod.reserve_slots(root_m, 1024)
        beams = [root_n] + [x for x in (nat.seq_fork(root_n) for _ in range(width - 1))]
        beams_m = [root_m] + [mod.seq_fork(root_m) for _ in range(width - 1)]
        assert beams == beams_m
        groups.append(beams)
    for step in range(20):
        for gi, beams in enumerate(groups):
            parents = [rnd.choice(beams) for _ in range(width)]
            kids_n = [nat.seq_fork(p) for p in parents]
            kids_m = [mod.seq_fork(p) for p in parents]
            assert kids_n == kids_m
            for b in beams:
                nat.seq_free(b)
                mod.seq_free(b)
            for k in kids_n:
                a = nat.reserve_slots(k, 1)
                b = mod.reserve_slots(k, 1)
                assert a[0] == b[0] and [tuple(p) for p in a[1]] == [tuple(p) for p in b[1]]
            groups[gi] = kids_n
        _same_state(nat, mod)


def test_errors_and_atomicity():
    nat = api.BlockManager(4, 16)
    s = nat.seq_create()
    nat.reserve_slots(s, 40)
    k = nat.seq_fork(s)
    free0, refs0 = nat.num_free(), [nat.refcount(b) for b in range(4)]
    with pytest.raises(api.NoFreeBlock):
        nat.reserve_slots(k, 1 + 2 * 16)
    assert nat.num_free() == free0 and [nat.refcount(b) for b in range(4)] == refs0
    with pytest.raises(api.PAError):
        nat.seq_free(99)
    with pytest.raises(api.PAError):
        nat.decref(3)                      # never allocated
    assert nat.refcount(-1) == -1 and nat.refcount(4) == -1
    with pytest.raises(api.PAError):
        nat.build_block_tables([s], 2)
    with pytest.raises(api.PAError):
        api.BlockManager(0, 16)


def test_batch_reservation_equals_sequential_calls():
    B = 16
    rnd = random.Random(11)
    nat, mod = api.BlockManager(4096, B), BlockManagerModel(4096, B)
    ids = []
    for i in range(40):
        a, b = nat.seq_create(), mod.seq_create()
        n = rnd.randint(1, 100)
        nat.reserve_slots(a, n)
        mod.reserve_slots(b, n)
        ids.append(a)
    for i in range(10):                      # some shared partial blocks -> copy-on-write
        p = rnd.choice(ids)
        ids.append(nat.seq_fork(p))
        mod.seq_fork(p)
    for step in range(5):
        slots, pairs = nat.reserve_slots_batch(ids, 1)
        ref_slots, ref_pairs = [], []
        for sid in ids:
            s_, p_ = mod.reserve_slots(sid, 1)
            ref_slots += s_
            ref_pairs += p_
        assert slots.tolist() == ref_slots
        assert [tuple(x) for x in pairs.tolist()] == [tuple(x) for x in ref_pairs]
    _same_state(nat, mod)


def test_batch_reservation_stops_at_first_failure():
    nat = api.BlockManager(3, 16)
    a, b = nat.seq_create(), nat.seq_create()
    nat.reserve_slots(a, 16)
    nat.reserve_slots(b, 16)
    c = nat.seq_create()
    with pytest.raises(api.NoFreeBlock):
        nat.reserve_slots_batch([a, b, c], 1)   # a gets the last block, b cannot
    assert nat.seq_len(a) == 17 and nat.seq_len(b) == 16 and nat.seq_len(c) == 0


def test_batched_fork_and_free_equal_single_calls():
    B = 16
    nat, mod = api.BlockManager(1024, B), BlockManagerModel(1024, B)
    roots = []
    for n in (40, 70, 16):
        a, b = nat.seq_create(), mod.seq_create()
        nat.reserve_slots(a, n)
        mod.reserve_slots(b, n)
        roots.append(a)
    parents = [roots[0], roots[0], roots[2], roots[1], roots[0]]
    kids = nat.seq_fork_batch(parents).tolist()
    assert kids == [mod.seq_fork(p) for p in parents]
    nat.seq_free_batch(roots)
    for r in roots:
        mod.seq_free(r)
    _same_state(nat, mod)
    with pytest.raises(api.PAError):
        nat.seq_free_batch([kids[0], 999])
    assert nat.seq_len(kids[0]) == -1          # freed before the unknown id stopped the batch


def test_batch_calls_check_their_host_arrays():
    # the batch calls hand plain addresses to the library: arrays it would write through must be
    # contiguous CPU tensors of the right type and size, and id arrays of another type are converted
    mgr = api.BlockManager(64, 16)
    seqs = [mgr.seq_create() for _ in range(4)]
    slots, pairs = mgr.reserve_slots_batch(torch.tensor(seqs, dtype=torch.int64), 3)   # ids converted
    assert slots.shape == (12,) and pairs.shape == (0, 2)
    with pytest.raises(ValueError):
        mgr.reserve_slots_batch(seqs, 1, torch.empty(4, dtype=torch.int32))             # wrong slot type
    with pytest.raises(ValueError):
        mgr.reserve_slots_batch(seqs, 2, torch.empty(4, dtype=torch.int64))             # too small
    with pytest.raises(ValueError):
        mgr.build_block_tables(seqs, 4, torch.empty((4, 4), dtype=torch.int32)[:, :2])  # not contiguous
    with pytest.raises(ValueError):
        mgr.build_block_tables(seqs, 4, None, torch.empty(4, dtype=torch.int64))        # wrong lens type
    tables, lens = mgr.build_block_tables(seqs, 4)
    assert lens.tolist() == [3, 3, 3, 3] and (tables[:, 0] >= 0).all() and (tables[:, 1:] == -1).all()
    kids = mgr.seq_fork_batch(torch.tensor(seqs, dtype=torch.int32)[::2])              # strided ids
    assert kids.tolist() == [4, 5]
    mgr.seq_free_batch(kids)
