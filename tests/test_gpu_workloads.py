"""GPU parity on the benchmark's own workloads, at their full sizes and partitions.

* Shared-prefix sampling and beam search (32 requests x 4 sequences over a 1024-token prompt whose
  64 blocks are shared at count 4; "PagedAttention原理", "解决共享prompt" and "解决COW"; "Paged
  Attention&Orca Paper笔记与解读", parallel sampling and beam search): the benchmark's own
  trajectory of beam-style forks, slot reservations with copy-on-write pairs, block copies, cache
  writes and decodes, run through the captured step (pa_step_*) at the library's default
  partition.  Every step's output is compared with the oracle applied to the state it reaches by
  replaying the same copies and writes; the caches are compared bit for bit at the end.
* The same with a 1031-token prompt: its last block holds 7 tokens and is shared by a request's
  four sequences, so the first step copies it for three of them and the fourth writes in place
  ("解决COW": N sharers writing once make N - 1 copies).
* Long contexts (16 sequences of 16-32 k tokens, 64/8 heads) at B = 8, 16 and 32 ("PagedAttention原理",
  "block_size 选取") for every partition size the benchmark's sweep uses, the library default included.

The block manager runs in lockstep with the oracle's model of it: every call is made on both and
must give identical ids, slots, pairs and tables, so the oracle side of each comparison takes its
tables, slots and pairs from the model, not from the library.

Tolerance: max-abs 2e-3 on fp32 outputs for bf16 caches (fp32 accumulation); block copies and
cache writes bit-exact.
"""
import pytest
import torch

import bench
from oracle.allocator import BlockManagerModel
from paged_kv_cache_329_b200 import api
from paged_kv_cache_329_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = 2e-3
_NativeManager = api.BlockManager


class _Lockstep:
    """api.BlockManager with the oracle's model run beside it (same calls, results must agree)."""

    def __init__(self, n_blocks, block_size):
        self.nat = _NativeManager(n_blocks, block_size)
        self.mod = BlockManagerModel(n_blocks, block_size)
        self.n_blocks, self.B = n_blocks, block_size
        self.last_slots, self.last_pairs, self.last_tables, self.last_lens = None, None, None, None

    def alloc_block(self):
        a, b = self.nat.alloc_block(), self.mod.alloc_block()
        assert a == b
        return a

    def decref(self, b):
        self.nat.decref(b)
        self.mod.decref(b)

    def refcount(self, b):
        a = self.nat.refcount(b)
        assert a == self.mod.refcount(b)
        return a

    def seq_create(self):
        a, b = self.nat.seq_create(), self.mod.seq_create()
        assert a == b
        return a

    def seq_fork(self, parent):
        a, b = self.nat.seq_fork(parent), self.mod.seq_fork(parent)
        assert a == b
        return a

    def reserve_slots(self, sid, n_new):
        got, want = self.nat.reserve_slots(sid, n_new), self.mod.reserve_slots(sid, n_new)
        assert got[0] == want[0] and [tuple(p) for p in got[1]] == [tuple(p) for p in want[1]]
        return got

    def seq_fork_batch(self, parents):
        kids = self.nat.seq_fork_batch(parents)
        assert kids.tolist() == [self.mod.seq_fork(int(p)) for p in parents]
        return kids

    def seq_free_batch(self, seq_ids):
        self.nat.seq_free_batch(seq_ids)
        for s in seq_ids.tolist():
            self.mod.seq_free(s)

    def reserve_slots_batch(self, seq_ids, n_new=1, slots=None, pairs=None):
        got_slots, got_pairs = self.nat.reserve_slots_batch(seq_ids, n_new, slots, pairs)
        want_slots, want_pairs = [], []
        for s in seq_ids.tolist():
            sl, pr = self.mod.reserve_slots(s, n_new)
            want_slots += sl
            want_pairs += [tuple(p) for p in pr]
        assert got_slots.tolist() == want_slots
        assert [tuple(p) for p in got_pairs.tolist()] == want_pairs
        self.last_slots = torch.tensor(want_slots, dtype=torch.int64)
        self.last_pairs = torch.tensor(want_pairs, dtype=torch.int32).reshape(-1, 2)
        return got_slots, got_pairs

    def build_block_tables(self, seq_ids, max_blocks_per_seq, tables=None, lens=None):
        t, l = self.nat.build_block_tables(seq_ids, max_blocks_per_seq, tables, lens)
        want_t, want_l = self.mod.build_block_tables(seq_ids.tolist(), max_blocks_per_seq)
        assert t.tolist() == want_t and l.tolist() == want_l
        self.last_tables = torch.tensor(want_t, dtype=torch.int32)
        self.last_lens = torch.tensor(want_l, dtype=torch.int32)
        return t, l


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_kv_cache_329_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _close(got, ref, what):
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got.double() - ref).abs().max().item()
    assert err <= TOL, f"{what}: max-abs error {err:.3g} > {TOL}"


def _trajectory(oracle_mod, monkeypatch, name, n_steps, check_first_step=None):
    monkeypatch.setattr(api, "BlockManager", _Lockstep)
    wl = bench.make_workload(name, torch.device("cuda"), growth_steps=n_steps + 2)
    mgr = wl.mgr
    assert isinstance(mgr, _Lockstep)
    S, H, Hk, d = wl.S, wl.H, wl.Hk, wl.d
    assert (S, H, Hk, d, wl.B) == (128, 32, 8, 128, 16)
    assert wl.P == api.default_partition(S, Hk, wl.max_c)
    step = api.DecodeStep(wl.k_cache, wl.v_cache, S, H, wl.max_blocks, wl.max_c, max_pairs=S,
                          out_dtype=torch.float32, partition_size=wl.P)
    k_ref, v_ref = wl.k_cache.cpu(), wl.v_cache.cpu()
    g = W.generator(4100)
    total_pairs = 0
    for it in range(n_steps):
        refs_before = None
        if it == 0 and check_first_step is not None:
            refs_before = {b: mgr.refcount(b) for b in set(mgr.mod.seqs[int(wl.seqs[0])]["table"])}
        wl.host_step(step.h_slots, None, step.h_tables, step.h_lens)
        pairs = mgr.last_pairs
        step.set_pairs(pairs)
        total_pairs += pairs.shape[0]
        if it == 0 and check_first_step is not None:
            check_first_step(wl, mgr, pairs, refs_before)
        q = W.randn(g, (S, H, d), wl.dtype)
        key = W.randn(g, (S, Hk, d), wl.dtype)
        val = W.randn(g, (S, Hk, d), wl.dtype)
        step.h_query.copy_(q)
        step.h_key.copy_(key)
        step.h_value.copy_(val)
        out = step.run().clone()
        # the oracle replays the step on its own state: copies, then writes, then decode
        k_ref, v_ref = oracle_mod.copy_blocks(k_ref, v_ref, pairs)
        k_ref, v_ref = oracle_mod.cache_write(k_ref, v_ref, key, val, mgr.last_slots)
        ref = oracle_mod.decode(q, k_ref, v_ref, mgr.last_tables, mgr.last_lens, n_threads=0)
        _close(out, ref, f"{name} step {it} (P={wl.P})")
        # the split-K path (partitions of 256 tokens, log-sum-exp combine) on the same device state
        out_split = api.pa_decode(step.d_query, wl.k_cache, wl.v_cache, step.d_tables, step.d_lens,
                                  max_context_len=wl.max_c, out_dtype=torch.float32, partition_size=256)
        torch.cuda.synchronize()
        _close(out_split.cpu(), ref, f"{name} step {it} (P=256)")
    assert api.workspace_error(step.workspace) == 0
    assert total_pairs > 0
    assert torch.equal(wl.k_cache.cpu().view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(wl.v_cache.cpu().view(torch.int16), v_ref.view(torch.int16))


def test_shared_prefix_trajectory_full_size(oracle_mod, monkeypatch):
    _trajectory(oracle_mod, monkeypatch, "shared_prefix_bf16", 6)


def test_shared_prefix_partial_prompt_block(oracle_mod, monkeypatch):
    def first_step(wl, mgr, pairs, refs_before):
        # Each request's 4 sequences share the 7-token last prompt block: 3 copies, 1 in-place write.
        partial = [b for b, r in refs_before.items() if r >= 4 and b in set(pairs[:, 0].tolist())]
        assert pairs.shape[0] == 3 * wl.REQUESTS
        srcs = pairs[:, 0].tolist()
        assert all(srcs.count(s) == 3 for s in set(srcs))
        assert len(set(srcs)) == wl.REQUESTS and len(partial) == 1
        assert all(mgr.refcount(s) == 1 for s in set(srcs))
        assert len(set(pairs[:, 1].tolist())) == pairs.shape[0]

    _trajectory(oracle_mod, monkeypatch, "shared_prefix_partial_bf16", 4, first_step)


def _oracle_sample(oracle_mod, case, seqs):
    q, bt, cl = case.q.cpu(), case.block_tables.cpu(), case.context_lens.cpu()
    seqs = torch.as_tensor(seqs)
    bt_s = bt[seqs]
    used = torch.unique(bt_s[bt_s >= 0])
    remap = torch.full((case.n_blocks,), -1, dtype=torch.int32)
    remap[used] = torch.arange(used.numel(), dtype=torch.int32)
    bt_r = torch.where(bt_s >= 0, remap[bt_s.clamp(min=0).long()], bt_s)
    kc = case.k_cache[used.to(case.k_cache.device)].cpu()
    vc = case.v_cache[used.to(case.v_cache.device)].cpu()
    return oracle_mod.decode(q[seqs], kc, vc, bt_r, cl[seqs], case.scale, n_threads=0)


@pytest.mark.parametrize("B", [8, 16, 32])
def test_long_context_every_partition(oracle_mod, B):
    case = W.long_bf16(B=B, device="cuda")
    lens = case.context_lens.cpu()
    sample = sorted({0, 7, int(torch.argmax(lens)), int(torch.argmin(lens))})
    ref = _oracle_sample(oracle_mod, case, sample)
    max_c = int(lens.max())
    assert api.default_partition(case.S, case.Hk, max_c) == 4096
    for P in (0, 512, 2048, 4096, 8192):
        ws = api.alloc_workspace(case.S, case.H, case.Hk, case.d, max_c, P)
        out = api.pa_decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                            max_context_len=max_c, scale=case.scale, out_dtype=torch.float32, partition_size=P,
                            workspace=ws)
        torch.cuda.synchronize()
        assert api.workspace_error(ws) == 0
        _close(out.cpu()[sample], ref, f"long B={B} P={P}")
        # bf16 output of the same call within one unit in the last place of the rounded oracle
        out16 = api.pa_decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              max_context_len=max_c, scale=case.scale, partition_size=P, workspace=ws).cpu()
        want = ref.to(torch.bfloat16)
        diff = (out16[sample].view(torch.int16).int() - want.view(torch.int16).int()).abs()
        assert bool(((diff <= 1) | ((out16[sample].double() - want.double()).abs() <= 1e-6)).all()), f"B={B} P={P}"
