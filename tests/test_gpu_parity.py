"""GPU parity of libpa's kernels against the fp64 oracle, through the C ABI.

Tolerances (max-abs, on fp32 outputs of the same kernels): 1e-5 for fp32 inputs, 2e-3 for fp16 and
bf16 inputs (fp32 accumulation).  Outputs in the input's 16-bit type are checked to within one
unit in the last place of the oracle's value rounded to that type.  Cache writes, block copies and
physical-permutation checks are bit-exact.
"""
import math

import pytest
import torch

from paged_kv_cache_329_b200 import api
from paged_kv_cache_329_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.float16: 2e-3, torch.bfloat16: 2e-3}


@pytest.fixture(params=["mma", "cuda_core"])
def consumer(request, monkeypatch):
    """16-bit caches: tensor-core consumers (default) or CUDA-core consumers."""
    monkeypatch.setenv("PA_DECODE_CONSUMER", request.param)
    return request.param


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from paged_kv_cache_329_b200 import build

    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _run(case: W.DecodeCase, out_dtype=torch.float32, P=0, max_c=None):
    dev = case.to("cuda") if not case.q.is_cuda else case
    if max_c is None:
        max_c = int(case.context_lens.max()) if case.S else 0
    ws = api.alloc_workspace(case.S, case.H, case.Hk, case.d, max_c, P)
    out = api.pa_decode(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                        max_context_len=max_c, scale=case.scale, out_dtype=out_dtype, partition_size=P,
                        workspace=ws)
    torch.cuda.synchronize()
    assert api.workspace_error(ws) == 0
    return out.cpu()


def _oracle(oracle_mod, case, seqs=None):
    """Oracle output for all sequences, or for a sample (gathering their blocks into a small pool)."""
    q, bt, cl = case.q.cpu(), case.block_tables.cpu(), case.context_lens.cpu()
    if seqs is None:
        return oracle_mod.decode(q, case.k_cache.cpu(), case.v_cache.cpu(), bt, cl, case.scale, n_threads=0)
    seqs = torch.as_tensor(seqs)
    bt_s = bt[seqs]
    used = torch.unique(bt_s[bt_s >= 0])
    remap = torch.full((case.n_blocks,), -1, dtype=torch.int32)
    remap[used] = torch.arange(used.numel(), dtype=torch.int32)
    bt_r = torch.where(bt_s >= 0, remap[bt_s.clamp(min=0).long()], bt_s)
    kc = case.k_cache[used.to(case.k_cache.device)].cpu()
    vc = case.v_cache[used.to(case.v_cache.device)].cpu()
    return oracle_mod.decode(q[seqs], kc, vc, bt_r, cl[seqs], case.scale, n_threads=0)


def _assert_close(got, ref, dtype, what=""):
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got.double() - ref).abs().max().item()
    assert err <= TOL[dtype], f"{what}: max-abs error {err:.3g} > {TOL[dtype]}"
    return err


def _assert_ulp(got, ref, what=""):
    """got: 16-bit output; ref: fp64 oracle.  |got - RNE(ref)| <= 1 ulp."""
    want = ref.to(got.dtype)
    gi = got.view(torch.int16).int()
    wi = want.view(torch.int16).int()
    ok = ((gi - wi).abs() <= 1) | ((got.double() - want.double()).abs() <= 1e-6)
    assert ok.all(), f"{what}: {(~ok).sum().item()} elements differ by more than 1 ulp"


# ---- the five serving scenarios ----------------------------------------------------------------

def test_tiny_fp32(oracle_mod):
    case = W.tiny_fp32()
    ref = _oracle(oracle_mod, case)
    _assert_close(_run(case), ref, torch.float32, "tiny_fp32")


def test_mha13b_fp16_with_cache_write(oracle_mod, consumer):
    case = W.mha13b_fp16()
    tables, lens, slots = W.new_token_slots(case, W.generator(102))
    g = W.generator(103)
    key = W.randn(g, (case.S, case.Hk, case.d), torch.float16)
    val = W.randn(g, (case.S, case.Hk, case.d), torch.float16)
    k_ref, v_ref = oracle_mod.cache_write(case.k_cache, case.v_cache, key, val, slots)
    dev = case.to("cuda")
    api.pa_cache_write(dev.k_cache, dev.v_cache, key.cuda(), val.cuda(), slots.cuda())
    torch.cuda.synchronize()
    assert torch.equal(dev.k_cache.cpu().view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(dev.v_cache.cpu().view(torch.int16), v_ref.view(torch.int16))
    grown = W.DecodeCase(case.name, case.q, k_ref, v_ref, tables, lens, case.scale, case.H, case.Hk, case.d, case.B)
    dev2 = W.DecodeCase(case.name, dev.q, dev.k_cache, dev.v_cache, tables.cuda(), lens.cuda(), case.scale,
                        case.H, case.Hk, case.d, case.B)
    ref = _oracle(oracle_mod, grown)
    _assert_close(_run(dev2, max_c=int(lens.max())), ref, torch.float16, "mha13b_fp16")
    _assert_ulp(_run(dev2, torch.float16, max_c=int(lens.max())), ref, "mha13b_fp16 fp16 out")


def test_gqa8k_bf16_full_size_sampled(oracle_mod, consumer):
    case = W.gqa8k_bf16(device="cuda")
    lens = case.context_lens.cpu()
    order = torch.argsort(lens)
    sample = torch.unique(torch.cat([order[:6], order[-6:], torch.arange(0, case.S, 23)]))
    ref = _oracle(oracle_mod, case, sample)
    got = _run(case)
    _assert_close(got[sample], ref, torch.bfloat16, "gqa8k_bf16")
    got16 = _run(case, torch.bfloat16)
    _assert_ulp(got16[sample], ref, "gqa8k_bf16 bf16 out")


@pytest.mark.parametrize("B", [8, 16, 32])
def test_long_context_full_size_sampled(oracle_mod, B, consumer):
    case = W.long_bf16(B=B, device="cuda")
    sample = [0, 7, int(torch.argmax(case.context_lens.cpu()))]
    ref = _oracle(oracle_mod, case, sample)
    for P in (256, 1024):
        got = _run(case, P=P)
        _assert_close(got[sample], ref, torch.bfloat16, f"long B={B} P={P}")


# ---- edge cases ----------------------------------------------------------------------------------

EDGE_LENS = [1, 7, 8, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 255, 256, 257, 511, 512, 513, 1100]


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B", [8, 16, 32])
def test_edge_lengths(oracle_mod, dtype, g, d, B, consumer):
    if dtype == torch.float32 and consumer == "cuda_core":
        pytest.skip("fp32 caches always use the CUDA-core consumers")
    Hk = 2
    case = W.paged_case("edge", EDGE_LENS, g * Hk, Hk, d, B, dtype, 1000 + g * 7 + d + B)
    ref = _oracle(oracle_mod, case)
    for P in (0, 64, 256):
        _assert_close(_run(case, P=P), ref, dtype, f"{dtype} g={g} d={d} B={B} P={P}")


def test_zero_length_sequences_give_zero(oracle_mod, consumer):
    case = W.paged_case("zero", [0, 5, 0, 300, 0], 8, 2, 128, 16, torch.bfloat16, 77)
    out = _run(case, P=64)
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0 and torch.count_nonzero(out[4]) == 0
    _assert_close(out, _oracle(oracle_mod, case), torch.bfloat16, "zero lengths")


def test_all_empty_batch():
    case = W.paged_case("empty", [0, 0], 4, 4, 64, 16, torch.float16, 78)
    assert torch.count_nonzero(_run(case)) == 0


def test_output_types(oracle_mod, consumer):
    case = W.paged_case("types", [3, 70, 600], 16, 4, 128, 16, torch.float16, 79)
    ref = _oracle(oracle_mod, case)
    _assert_close(_run(case, torch.float32), ref, torch.float16, "f32 out")
    _assert_ulp(_run(case, torch.float16), ref, "f16 out")
    _assert_ulp(_run(case, torch.bfloat16), ref, "bf16 out")


# ---- determinism and placement -----------------------------------------------------------------

@pytest.mark.parametrize("B", [8, 16, 32])
def test_physical_permutation_is_bit_identical(B, consumer):
    case = W.paged_case("perm", [1, B + 1, 200, 700, 1500], 32, 8, 128, B, torch.bfloat16, 80 + B, pool_factor=2.0)
    o1 = _run(case, P=256)
    n = case.n_blocks
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(B))
    kc2 = torch.empty_like(case.k_cache)
    vc2 = torch.empty_like(case.v_cache)
    kc2[perm] = case.k_cache
    vc2[perm] = case.v_cache
    bt2 = case.block_tables.clone()
    m = bt2 >= 0
    bt2[m] = perm[bt2[m].long()].to(torch.int32)
    case2 = W.DecodeCase("perm2", case.q, kc2, vc2, bt2, case.context_lens, case.scale, case.H, case.Hk, case.d, B)
    o2 = _run(case2, P=256)
    assert torch.equal(o1, o2)
    assert torch.equal(o1, _run(case, P=256))  # and a repeat call


def test_split_and_unsplit_agree(oracle_mod, consumer):
    case = W.paged_case("split", [2000, 3000, 64, 4097], 32, 8, 128, 16, torch.bfloat16, 90)
    ref = _oracle(oracle_mod, case)
    outs = [_run(case, P=P) for P in (64, 512, 4160)]   # 4160 >= every length: no split at all
    for o in outs:
        _assert_close(o, ref, torch.bfloat16, "split")
    assert (outs[0] - outs[2]).abs().max() < 1e-4


def test_shared_prefix_reads_same_blocks(oracle_mod, consumer):
    # Sequences whose tables share the prompt blocks and whose tails and queries match produce
    # identical outputs.
    case = W.paged_case("pref", [1030, 1030], 32, 8, 128, 16, torch.bfloat16, 91, sentinel="none", n_blocks=200)
    bt = case.block_tables.clone()
    bt[1, :64] = bt[0, :64]
    kc, vc = case.k_cache.clone(), case.v_cache.clone()
    kc[int(bt[1, 64])] = kc[int(bt[0, 64])]
    vc[int(bt[1, 64])] = vc[int(bt[0, 64])]
    q = case.q.clone()
    q[1] = q[0]
    c2 = W.DecodeCase("pref2", q, kc, vc, bt, case.context_lens, case.scale, case.H, case.Hk, case.d, case.B)
    out = _run(c2)
    assert torch.equal(out[0], out[1])
    _assert_close(out, _oracle(oracle_mod, c2), torch.bfloat16, "shared prefix")


# ---- combine, cache write, copy blocks ---------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("long", [False, True])   # True: more than 64 partitions (several warps per row)
def test_combine_matches_oracle(oracle_mod, d, long):
    P = 64
    lens = torch.tensor([1, 64, 65, 300, 0, 6000 if long else 1000] + ([4160, 2111, 64 * 70] if long else []),
                        dtype=torch.int32)
    case = W.paged_case("comb", lens, 8, 2, d, 16, torch.float32, 92)
    n_parts = int(math.ceil(int(lens.max()) / P))
    po, pm, pl = oracle_mod.partials(case.q, case.k_cache, case.v_cache, case.block_tables, lens, P, n_parts)
    po32, pm32, pl32 = po.float(), pm.float(), pl.float()
    ref = oracle_mod.combine(po32, pm32, pl32)
    got = api.pa_combine(po32.cuda(), pm32.cuda(), pl32.cuda(), lens.cuda(), P).cpu()
    assert torch.isfinite(got).all()
    assert (got.double() - ref).abs().max() < 1e-5
    assert torch.count_nonzero(got[4]) == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("d,B", [(64, 8), (128, 16), (128, 32)])
def test_cache_write_bit_exact(oracle_mod, dtype, d, B):
    n_blocks, Hk, T = 40, 4, 75
    g = W.generator(200 + d + B)
    kc = W.randn(g, (n_blocks, Hk, B, d), dtype)
    vc = W.randn(g, (n_blocks, Hk, B, d), dtype)
    key = W.randn(g, (T, Hk, d), dtype)
    val = W.randn(g, (T, Hk, d), dtype)
    slots = torch.randperm(n_blocks * B, generator=g)[:T].to(torch.int64)
    slots[::9] = -1
    k_ref, v_ref = oracle_mod.cache_write(kc, vc, key, val, slots)
    kd, vd = kc.cuda(), vc.cuda()
    api.pa_cache_write(kd, vd, key.cuda(), val.cuda(), slots.cuda())
    torch.cuda.synchronize()
    bits = torch.int32 if dtype == torch.float32 else torch.int16
    assert torch.equal(kd.cpu().view(bits), k_ref.view(bits))
    assert torch.equal(vd.cpu().view(bits), v_ref.view(bits))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_copy_blocks_bit_exact(oracle_mod, dtype):
    n_blocks, Hk, B, d = 64, 8, 16, 128
    g = W.generator(300)
    kc = W.randn(g, (n_blocks, Hk, B, d), dtype)
    vc = W.randn(g, (n_blocks, Hk, B, d), dtype)
    perm = torch.randperm(n_blocks, generator=g)
    pairs = torch.stack([perm[:20], perm[20:40]], 1).to(torch.int32)  # distinct dsts, no dst is a src
    k_ref, v_ref = oracle_mod.copy_blocks(kc, vc, pairs)
    kd, vd = kc.cuda(), vc.cuda()
    api.pa_copy_blocks(kd, vd, pairs.cuda())
    torch.cuda.synchronize()
    bits = torch.int32 if dtype == torch.float32 else torch.int16
    assert torch.equal(kd.cpu().view(bits), k_ref.view(bits))
    assert torch.equal(vd.cpu().view(bits), v_ref.view(bits))


# ---- the fused decode step (pa_decode_step) -----------------------------------------------------------

@pytest.mark.parametrize("dtype,B,d,g", [(torch.bfloat16, 16, 128, 4), (torch.float16, 8, 128, 1),
                                         (torch.float32, 32, 64, 2), (torch.bfloat16, 8, 64, 8)])
def test_decode_step_matches_copy_write_decode(oracle_mod, dtype, B, d, g):
    # Sequences forked from shared parents reserve 1-3 new tokens each (copy-on-write pairs where a
    # shared last block has room), plus padding tokens (slot -1).  The block manager is the
    # oracle's model; pa_decode_step must equal copy -> write -> decode by the oracle, with the
    # pair count read on the device and garbage rows past it ignored.
    from oracle.allocator import BlockManagerModel

    Hk, n_blocks = 2, 600
    H = g * Hk
    mgr = BlockManagerModel(n_blocks, B)
    rnd = torch.Generator().manual_seed(800 + B + d)
    roots = []
    for i in range(6):
        r = mgr.seq_create()
        mgr.reserve_slots(r, int(torch.randint(1, 300, (1,), generator=rnd)))
        roots.append(r)
    seqs = []
    for r in roots:
        seqs += [r] + [mgr.seq_fork(r) for _ in range(int(torch.randint(0, 4, (1,), generator=rnd)))]
    slots, pairs = [], []
    for s_ in seqs:
        n_new = int(torch.randint(1, 4, (1,), generator=rnd))
        sl, pr = mgr.reserve_slots(s_, n_new)
        slots += sl + ([-1] if n_new == 2 else [])
        pairs += pr
    assert len(pairs) > 0
    tables, lens = mgr.build_block_tables(seqs, max(len(mgr.seq_table(x)) for x in seqs))
    tables, lens = torch.tensor(tables, dtype=torch.int32), torch.tensor(lens, dtype=torch.int32)
    slots = torch.tensor(slots, dtype=torch.int64)
    T, S = slots.numel(), len(seqs)
    g_in = W.generator(801 + B)
    kc = W.randn(g_in, (n_blocks, Hk, B, d), dtype)
    vc = W.randn(g_in, (n_blocks, Hk, B, d), dtype)
    key = W.randn(g_in, (T, Hk, d), dtype)
    val = W.randn(g_in, (T, Hk, d), dtype)
    q = W.randn(g_in, (S, H, d), dtype)
    pr = torch.tensor(pairs, dtype=torch.int32).reshape(-1, 2)
    # rows past the count: copies that would overwrite live blocks if they were made
    assert int(tables[0, 0]) != int(tables[-1, 0])
    padded = torch.cat([pr, torch.tensor([[int(tables[0, 0]), int(tables[-1, 0])]] * 5, dtype=torch.int32)])
    n_dev = torch.tensor([pr.shape[0]], dtype=torch.int32, device="cuda")
    k_ref, v_ref = oracle_mod.copy_blocks(kc, vc, pr)
    k_ref, v_ref = oracle_mod.cache_write(k_ref, v_ref, key, val, slots)
    ref = oracle_mod.decode(q, k_ref, v_ref, tables, lens, 1.0 / math.sqrt(d))
    kd, vd = kc.cuda(), vc.cuda()
    max_c = int(lens.max())
    for P in (0, 64):
        kd.copy_(kc.cuda())
        vd.copy_(vc.cuda())
        ws = api.alloc_workspace(S, H, Hk, d, max_c, P)
        out = api.pa_decode_step(q.cuda(), kd, vd, tables.cuda(), lens.cuda(), key.cuda(), val.cuda(), slots.cuda(),
                                 padded.cuda(), n_pairs=n_dev, max_context_len=max_c, out_dtype=torch.float32,
                                 partition_size=P, workspace=ws)
        torch.cuda.synchronize()
        assert api.workspace_error(ws) == 0
        bits = torch.int32 if dtype == torch.float32 else torch.int16
        assert torch.equal(kd.cpu().view(bits), k_ref.view(bits)), f"K cache P={P}"
        assert torch.equal(vd.cpu().view(bits), v_ref.view(bits)), f"V cache P={P}"
        _assert_close(out.cpu(), ref, dtype, f"decode step {dtype} B={B} d={d} g={g} P={P}")
    # the pair count given on the host instead (no device count): the same result
    kd.copy_(kc.cuda())
    vd.copy_(vc.cuda())
    out = api.pa_decode_step(q.cuda(), kd, vd, tables.cuda(), lens.cuda(), key.cuda(), val.cuda(), slots.cuda(),
                             pr.cuda(), max_context_len=max_c, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _assert_close(out.cpu(), ref, dtype, "decode step, host count")


def test_decode_step_without_pairs_or_tokens(oracle_mod):
    case = W.paged_case("step0", [5, 300, 0, 64], 8, 2, 128, 16, torch.bfloat16, 810)
    dev = case.to("cuda")
    none_i32 = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    key = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    slots = torch.empty((0,), dtype=torch.int64, device="cuda")
    out = api.pa_decode_step(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens, key, key, slots,
                             none_i32, max_context_len=300, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _assert_close(out.cpu(), _oracle(oracle_mod, case), torch.bfloat16, "step without pairs or tokens")


# ---- the captured step (pa_step_*) ------------------------------------------------------------------

@pytest.mark.parametrize("max_pairs", [None, 9000])
def test_captured_step_matches_separate_calls(oracle_mod, max_pairs):
    # Shared-prefix trajectory: forks create copy-on-write pairs every step.  Each replay of the
    # graph must equal the oracle applied to the same block manager state.  With room for more
    # pairs than the fused step's prologue takes, the graph holds the copy, write and decode calls
    # instead (the pair count still read on the device).
    B, H, Hk, d, dt = 16, 32, 8, 128, torch.bfloat16
    mgr = api.BlockManager(512, B)
    g = W.generator(400)
    kc = W.randn(g, (512, Hk, B, d), dt)
    vc = W.randn(g, (512, Hk, B, d), dt)
    roots = []
    for r in range(4):
        root = mgr.seq_create()
        mgr.reserve_slots(root, 200 + 13 * r)
        roots.append([root] + [mgr.seq_fork(root) for _ in range(3)])
    kd, vd = kc.cuda(), vc.cuda()
    S = 16
    step = api.DecodeStep(kd, vd, S, H, 32, 512, out_dtype=torch.float32,
                          **({} if max_pairs is None else {"max_pairs": max_pairs}))
    k_ref, v_ref = kc.clone(), vc.clone()
    rnd = torch.Generator().manual_seed(9)
    for it in range(3):
        seqs = []
        for gi, beams in enumerate(roots):
            parents = torch.randint(0, 4, (4,), generator=rnd).tolist()
            kids = [mgr.seq_fork(beams[p]) for p in parents]
            for b in beams:
                mgr.seq_free(b)
            roots[gi] = kids
            seqs += kids
        slots, pairs = mgr.reserve_slots_batch(seqs, 1, step.h_slots)
        mgr.build_block_tables(seqs, 32, step.h_tables, step.h_lens)
        step.set_pairs(pairs)
        step.h_query.copy_(W.randn(g, (S, H, d), dt))
        step.h_key.copy_(W.randn(g, (S, Hk, d), dt))
        step.h_value.copy_(W.randn(g, (S, Hk, d), dt))
        out = step.run().clone()
        k_ref, v_ref = oracle_mod.copy_blocks(k_ref, v_ref, pairs)
        k_ref, v_ref = oracle_mod.cache_write(k_ref, v_ref, step.h_key, step.h_value, step.h_slots)
        ref = oracle_mod.decode(step.h_query, k_ref, v_ref, step.h_tables, step.h_lens)
        assert pairs.shape[0] > 0 or it > 0
        _assert_close(out, ref, dt, f"captured step {it}")
    # the same graph enqueued without waiting (launch): the last step again, whose copies and writes
    # repeat the same bytes, gives the same output once the stream has reached it
    step.h_out.zero_()
    step.launch(torch.cuda.current_stream())
    torch.cuda.current_stream().synchronize()
    _assert_close(step.h_out.clone(), ref, dt, "captured step, launch()")
    assert torch.equal(kd.cpu().view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(vd.cpu().view(torch.int16), v_ref.view(torch.int16))
    assert api.workspace_error(step.workspace) == 0


def test_pipelined_steps_match_oracle(oracle_mod):
    # Two captured steps launched alternately with launch_async: step i+1's input copy and step
    # i-1's output copy overlap step i's kernels.  Every output must equal the oracle applied to the
    # block manager state of its own step, and the caches must end bit-identical.
    B, H, Hk, d, dt = 16, 32, 8, 128, torch.bfloat16
    mgr = api.BlockManager(512, B)
    g = W.generator(410)
    kc = W.randn(g, (512, Hk, B, d), dt)
    vc = W.randn(g, (512, Hk, B, d), dt)
    roots = []
    for r in range(4):
        root = mgr.seq_create()
        mgr.reserve_slots(root, 150 + 29 * r)
        roots.append([root] + [mgr.seq_fork(root) for _ in range(3)])
    kd, vd = kc.cuda(), vc.cuda()
    S = 16
    steps = [api.DecodeStep(kd, vd, S, H, 32, 512, out_dtype=torch.float32) for _ in range(2)]
    k_ref, v_ref = kc.clone(), vc.clone()
    rnd = torch.Generator().manual_seed(11)
    stream = torch.cuda.current_stream()
    refs = {}
    n_steps = 7
    for it in range(n_steps):
        step = steps[it % 2]
        if it >= 2:
            _assert_close(step.wait().clone(), refs.pop(it - 2), dt, f"pipelined step {it - 2}")
        seqs = []
        for gi, beams in enumerate(roots):
            parents = torch.randint(0, 4, (4,), generator=rnd).tolist()
            kids = [mgr.seq_fork(beams[p]) for p in parents]
            for b in beams:
                mgr.seq_free(b)
            roots[gi] = kids
            seqs += kids
        slots, pairs = mgr.reserve_slots_batch(seqs, 1, step.h_slots)
        mgr.build_block_tables(seqs, 32, step.h_tables, step.h_lens)
        step.set_pairs(pairs)
        step.h_query.copy_(W.randn(g, (S, H, d), dt))
        step.h_key.copy_(W.randn(g, (S, Hk, d), dt))
        step.h_value.copy_(W.randn(g, (S, Hk, d), dt))
        step.launch_async(stream)
        k_ref, v_ref = oracle_mod.copy_blocks(k_ref, v_ref, pairs)
        k_ref, v_ref = oracle_mod.cache_write(k_ref, v_ref, step.h_key, step.h_value, step.h_slots)
        refs[it] = oracle_mod.decode(step.h_query, k_ref, v_ref, step.h_tables, step.h_lens)
    for it in (n_steps - 2, n_steps - 1):
        _assert_close(steps[it % 2].wait().clone(), refs.pop(it), dt, f"pipelined step {it}")
    torch.cuda.synchronize()
    assert torch.equal(kd.cpu().view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(vd.cpu().view(torch.int16), v_ref.view(torch.int16))
    assert all(api.workspace_error(st.workspace) == 0 for st in steps)


# ---- swap to pinned host memory and back (pa_swap_blocks) --------------------------------------------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_swap_out_and_in_bit_exact(oracle_mod, dtype):
    n_dev, n_host, Hk, B, d = 48, 20, 8, 16, 128
    g = W.generator(500)
    dev_k = W.randn(g, (n_dev, Hk, B, d), dtype)
    dev_v = W.randn(g, (n_dev, Hk, B, d), dtype)
    host_k = W.randn(g, (n_host, Hk, B, d), dtype).pin_memory()
    host_v = W.randn(g, (n_host, Hk, B, d), dtype).pin_memory()
    out_pairs = torch.tensor([[3, 0], [17, 9], [40, 19], [8, 4]], dtype=torch.int32)
    ref_hk, ref_hv = oracle_mod.swap_blocks(host_k, host_v, dev_k, dev_v, out_pairs)
    dk, dv = dev_k.cuda(), dev_v.cuda()
    api.pa_swap_blocks(host_k, host_v, dk, dv, out_pairs.cuda())          # device -> pinned host
    torch.cuda.synchronize()
    bits = torch.int32 if dtype == torch.float32 else torch.int16
    assert torch.equal(host_k.view(bits), ref_hk.view(bits)) and torch.equal(host_v.view(bits), ref_hv.view(bits))
    in_pairs = torch.tensor([[0, 30], [9, 31], [19, 5], [4, 47]], dtype=torch.int32).pin_memory()
    ref_dk, ref_dv = oracle_mod.swap_blocks(dev_k, dev_v, ref_hk, ref_hv, in_pairs)
    api.pa_swap_blocks(dk, dv, host_k, host_v, in_pairs)                  # pinned host -> device
    torch.cuda.synchronize()
    assert torch.equal(dk.cpu().view(bits), ref_dk.view(bits)) and torch.equal(dv.cpu().view(bits), ref_dv.view(bits))


# ---- prefill chunks and mixed batches (pa_prefill) ---------------------------------------------------

def _prefill_case(ctx, nq, H, Hk, d, B, dtype, seed):
    case = W.paged_case("prefill", ctx, H, Hk, d, B, dtype, seed)
    q_start = torch.tensor([0] + list(torch.tensor(nq).cumsum(0)), dtype=torch.int32)
    q = W.randn(W.generator(seed + 7), (int(q_start[-1]), H, d), dtype)
    return case, q, q_start


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B", [8, 16, 32])
def test_prefill_mixed_batch(oracle_mod, dtype, g, d, B):
    # decode rows (n = 1), short and long chunks, chunks starting mid-context and whole prompts
    ctx = [1, 40, 77, 200, 300, 513, 64]
    nq = [1, 1, 77, 17, 129, 70, 64]
    Hk = 2
    case, q, q_start = _prefill_case(ctx, nq, g * Hk, Hk, d, B, dtype, 600 + g + d + B)
    ref = oracle_mod.prefill(q, q_start, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                             case.scale, n_threads=0)
    dev = case.to("cuda")
    ws = torch.empty(api.prefill_workspace_size(case.S, case.H, Hk, d, max(ctx), max(nq)), dtype=torch.uint8,
                     device="cuda")
    out = api.pa_prefill(q.cuda(), q_start.cuda(), dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                         max_context_len=max(ctx), max_q_len=max(nq), scale=case.scale, out_dtype=torch.float32,
                         workspace=ws)
    torch.cuda.synchronize()
    assert api.workspace_error(ws) == 0
    _assert_close(out.cpu(), ref, dtype, f"prefill {dtype} g={g} d={d} B={B}")


@pytest.mark.parametrize("dtype,d,g", [(torch.float16, 128, 4), (torch.bfloat16, 128, 4), (torch.bfloat16, 128, 8),
                                       (torch.bfloat16, 64, 1), (torch.bfloat16, 64, 8)])
def test_prefill_many_units_per_cta(oracle_mod, dtype, d, g):
    # about ten work units per persistent CTA, so that the tile counter, the S/P buffer parity and
    # the barrier phases run on across units: short chunks (one 64-key tile up to several, odd and
    # even tile counts), chunks that leave the second 128-row half without a query (at most 128 / g
    # tokens) next to ones that fill both halves, and decode rows; d = 64 has one 128-byte panel and
    # a deeper K/V ring
    gen = W.generator(690 + g + d)
    S = 700 if g <= 4 else 400
    nq = torch.randint(2, 256 // g + 8, (S,), generator=gen)
    nq[::9] = 1
    ctx = (nq + torch.randint(0, 230, (S,), generator=gen)).tolist()
    nq = nq.tolist()
    case, q, q_start = _prefill_case(ctx, nq, 2 * g, 2, d, 16, dtype, 691)
    ref = oracle_mod.prefill(q, q_start, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                             case.scale, n_threads=0)
    dev = case.to("cuda")
    ws = torch.empty(api.prefill_workspace_size(case.S, case.H, 2, d, max(ctx), max(nq)), dtype=torch.uint8,
                     device="cuda")
    for _ in range(2):  # twice in a row: the second call reuses the workspace the first one left
        out = api.pa_prefill(q.cuda(), q_start.cuda(), dev.k_cache, dev.v_cache, dev.block_tables,
                             dev.context_lens, max_context_len=max(ctx), max_q_len=max(nq), scale=case.scale,
                             out_dtype=torch.float32, workspace=ws)
        torch.cuda.synchronize()
        assert api.workspace_error(ws) == 0
        _assert_close(out.cpu(), ref, dtype, f"prefill, many units per CTA, {dtype} d={d} g={g}")


@pytest.fixture(params=["tcgen05", "mma_sync"])
def prefill_consumer(request, monkeypatch):
    """pa_prefill consumers: tcgen05 with TMEM accumulators (default) or mma.sync."""
    if request.param == "mma_sync":
        monkeypatch.setenv("PA_PREFILL_CONSUMER", "mma_sync")
    else:
        monkeypatch.delenv("PA_PREFILL_CONSUMER", raising=False)
    return request.param


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("scale", [-0.3, 0.0, 0.125, 0.3, 1.0])
def test_prefill_scale_sign(oracle_mod, prefill_consumer, dtype, scale):
    # the softmax of scale * q.k for a negative scale (the largest weight on the smallest score),
    # for scale 0 (the mean of the visible values), and for large scales whose wide score spread
    # makes the running maximum grow by more than 2^8 often (rescaling the accumulated output);
    # ragged chunks, decode rows, g = 4
    ctx, nq = [300, 77, 513, 1], [129, 77, 1, 1]
    case, q, q_start = _prefill_case(ctx, nq, 8, 2, 128, 16, dtype, 640)
    ref = oracle_mod.prefill(q, q_start, case.k_cache, case.v_cache, case.block_tables, case.context_lens, scale,
                             n_threads=0)
    dev = case.to("cuda")
    out = api.pa_prefill(q.cuda(), q_start.cuda(), dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                         max_context_len=max(ctx), max_q_len=max(nq), scale=scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _assert_close(out.cpu(), ref, dtype, f"prefill {prefill_consumer} scale={scale}")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("g", [1, 8])
def test_prefill_mixed_batch_mma_sync(oracle_mod, monkeypatch, dtype, g):
    monkeypatch.setenv("PA_PREFILL_CONSUMER", "mma_sync")
    test_prefill_mixed_batch(oracle_mod, dtype, g, 128, 16)


@pytest.mark.parametrize("scale", [-0.2, 0.0])
def test_decode_scale_sign(oracle_mod, consumer, scale):
    case = W.paged_case("dec-scale", [1, 17, 300, 1000], 8, 2, 128, 16, torch.bfloat16, 660)
    ref = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, scale)
    dev = case.to("cuda")
    out = api.pa_decode(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                        max_context_len=1000, scale=scale, out_dtype=torch.float32, partition_size=256)
    torch.cuda.synchronize()
    _assert_close(out.cpu(), ref, torch.bfloat16, f"decode {consumer} scale={scale}")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_prefill_edge_chunks(oracle_mod, prefill_consumer, dtype):
    # sequences with no query token beside ones that have some; chunks of exactly one 64-key tile,
    # one past it, exactly one 256-row unit (g = 4: 64 tokens) and one past it; whole prompts
    # (context = chunk) and a chunk whose context ends on a block boundary
    ctx = [50, 64, 65, 128, 129, 256, 300, 16]
    nq = [0, 64, 65, 64, 65, 256, 0, 16]
    case, q, q_start = _prefill_case(ctx, nq, 8, 2, 128, 16, dtype, 670)
    ref = oracle_mod.prefill(q, q_start, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                             case.scale, n_threads=0)
    dev = case.to("cuda")
    out = api.pa_prefill(q.cuda(), q_start.cuda(), dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                         max_context_len=max(ctx), max_q_len=max(nq), scale=case.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _assert_close(out.cpu(), ref, dtype, f"prefill edge chunks {prefill_consumer}")


def test_prefill_without_queries_and_empty_decode_batch():
    # every sequence contributes context but no query token: nothing to compute, no error
    case, q, q_start = _prefill_case([40, 7], [0, 0], 8, 2, 64, 16, torch.bfloat16, 671)
    dev = case.to("cuda")
    q0 = torch.empty((0, 8, 64), dtype=torch.bfloat16, device="cuda")
    out = api.pa_prefill(q0, q_start.cuda(), dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                         max_context_len=40, max_q_len=0)
    torch.cuda.synchronize()
    assert out.shape == (0, 8, 64)
    # a decode batch of no sequence
    case2 = W.paged_case("s0", [5], 8, 2, 64, 16, torch.bfloat16, 672).to("cuda")
    out2 = api.pa_decode(case2.q[:0], case2.k_cache, case2.v_cache, case2.block_tables[:0], case2.context_lens[:0],
                         max_context_len=5)
    torch.cuda.synchronize()
    assert out2.shape == (0, 8, 64)


def test_prefill_single_tokens_match_decode():
    case = W.gqa8k_bf16(S=32)
    dev = case.to("cuda")
    q_start = torch.arange(case.S + 1, dtype=torch.int32, device="cuda")
    max_c = int(case.context_lens.max())
    out_p = api.pa_prefill(dev.q, q_start, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                           max_context_len=max_c, max_q_len=1, out_dtype=torch.float32)
    out_d = api.pa_decode(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                          max_context_len=max_c, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert (out_p - out_d).abs().max().item() < 2e-3


def test_prefill_long_prompt_sampled(oracle_mod):
    # one 2048-token prompt chunk at the end of a 6000-token context, GQA 32/8, bf16
    ctx, nq = [6000, 3000], [2048, 1]
    case, q, q_start = _prefill_case(ctx, nq, 32, 8, 128, 16, torch.bfloat16, 650)
    dev = case.to("cuda")
    out = api.pa_prefill(q.cuda(), q_start.cuda(), dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                         max_context_len=6000, max_q_len=2048, scale=case.scale, out_dtype=torch.float32).cpu()
    rows = torch.tensor([0, 1, 63, 64, 1000, 2046, 2047, 2048])
    # oracle on the sampled rows: cut each row's context at its position and decode it
    for r in rows.tolist():
        s = 0 if r < 2048 else 1
        pos = ctx[s] - nq[s] + (r - int(q_start[s]))
        lens = case.context_lens.clone()
        lens[s] = pos + 1
        ref = oracle_mod.decode(q[r:r + 1].expand(2, -1, -1).contiguous(), case.k_cache, case.v_cache,
                                case.block_tables, lens, case.scale)[s]
        _assert_close(out[r], ref, torch.bfloat16, f"prefill row {r}")



# ---- failure detection without a GPU fault ------------------------------------------------------------

def test_bounded_wait_gives_up_and_context_survives():
    import time as _time
    lib = api._native.load()
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    t0 = _time.time()
    assert lib.pa_selftest_wait_timeout(50000, api._ptr(status), None) == api.PA_OK   # 50 ms
    torch.cuda.synchronize()
    assert int(status) == 2                      # the wait ran out and said so
    assert _time.time() - t0 < 5.0
    case = W.paged_case("after", [100, 7], 8, 2, 64, 16, torch.bfloat16, 700)
    assert torch.isfinite(_run(case)).all()     # the context still runs kernels


def test_out_of_range_block_id_is_reported_not_faulted(oracle_mod):
    # A bad table entry reads as zeros (the TMA unit fills a box outside the tensor) and sets bit 0
    # of the error word; every other sequence is unaffected.
    case = W.paged_case("badblk", [40, 100, 33], 8, 2, 128, 16, torch.bfloat16, 701, sentinel="none")
    bt = case.block_tables.clone()
    bt[1, 2] = case.n_blocks + 5                 # out of range
    dev = W.DecodeCase("badblk", case.q, case.k_cache, case.v_cache, bt, case.context_lens, case.scale,
                       case.H, case.Hk, case.d, case.B).to("cuda")
    ws = api.alloc_workspace(case.S, case.H, case.Hk, case.d, 100, 64)
    out = api.pa_decode(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens, max_context_len=100,
                        scale=case.scale, out_dtype=torch.float32, partition_size=64, workspace=ws).cpu()
    assert api.workspace_error(ws) & 1
    ref = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    _assert_close(out[[0, 2]], ref[[0, 2]], torch.bfloat16, "other sequences")
    assert torch.isfinite(out[1]).all()
