"""Pins for the attention oracle: checks against closed forms, invariants, an independent library
routine and the block-wise formulation -- never against the oracle itself.

Each test names the passage it follows (page title, section, equation).
"""
import math
import random

import pytest
import torch

from paged_kv_cache_329_b200 import workloads as W

DT = [torch.float32, torch.float16, torch.bfloat16]


# ---- element decoding (a library routine: torch's own conversion) ---------------------------------

@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_elem_decoding_matches_torch(oracle_mod, dtype):
    bits = torch.arange(0, 1 << 16, 97, dtype=torch.int32).to(torch.int16)
    # include subnormals, zero, infinities
    special = torch.tensor([0, 1, 0x3FF, 0x400, 0x7C00, -0x8000 + 1, 0x7F80, 0x0080], dtype=torch.int32).to(torch.int16)
    bits = torch.cat([bits, special])
    vals = bits.view(dtype)
    ref = vals.to(torch.float64)
    for i in range(bits.numel()):
        a = oracle_mod.elem_to_double(vals, i)
        b = float(ref[i])
        assert (math.isnan(a) and math.isnan(b)) or a == b, (i, a, b)


# ---- closed forms of o_t = softmax(q_t K^T / sqrt(d)) V  ("PagedAttention原理", 为什么会有 KV cache) ----

@pytest.mark.parametrize("dtype", DT)
def test_single_token_returns_its_value(oracle_mod, dtype):
    # c = 1: the softmax has one weight, equal to 1, so o = v_0 exactly.
    case = W.paged_case("c1", [1, 1, 1], 4, 2, 64, 16, dtype, 11)
    o = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    for s in range(3):
        blk = int(case.block_tables[s, 0])
        for h in range(4):
            v0 = case.v_cache[blk, h // 2, 0].to(torch.float64)
            assert torch.equal(o[s, h], v0)


def test_equal_keys_give_mean_of_values(oracle_mod):
    # All scores equal -> uniform weights 1/c -> o = mean of the values.
    c, d, B = 37, 64, 8
    case = W.paged_case("eqk", [c], 2, 1, d, B, torch.float32, 12)
    kc = case.k_cache.clone()
    kvec = torch.randn(d)
    for j in range((c + B - 1) // B):
        kc[int(case.block_tables[0, j])] = kvec
    o = oracle_mod.decode(case.q, kc, case.v_cache, case.block_tables, case.context_lens)
    vs = torch.stack([case.v_cache[int(case.block_tables[0, t // B]), 0, t % B].double() for t in range(c)])
    assert torch.allclose(o[0, 0], vs.mean(0), atol=1e-13, rtol=0)
    assert torch.allclose(o[0, 1], vs.mean(0), atol=1e-13, rtol=0)


def test_zero_query_gives_mean_of_values(oracle_mod):
    c, d, B = 50, 128, 16
    case = W.paged_case("q0", [c], 1, 1, d, B, torch.bfloat16, 13)
    q = torch.zeros_like(case.q)
    o = oracle_mod.decode(q, case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    vs = torch.stack([case.v_cache[int(case.block_tables[0, t // B]), 0, t % B].double() for t in range(c)])
    assert torch.allclose(o[0, 0], vs.mean(0), atol=1e-13, rtol=0)


def test_three_token_closed_form(oracle_mod):
    # d = 1, scale 1, q = 1, keys (0, 1, 2), values (0, 0, 1):
    # o = e^2 / (1 + e + e^2).  Keys sit in two blocks of B = 2 at physical ids (3, 1).
    kc = torch.full((4, 1, 2, 1), float("nan"), dtype=torch.float64).float()
    vc = kc.clone()
    kc[3, 0, 0, 0], kc[3, 0, 1, 0], kc[1, 0, 0, 0] = 0.0, 1.0, 2.0
    vc[3, 0, 0, 0], vc[3, 0, 1, 0], vc[1, 0, 0, 0] = 0.0, 0.0, 1.0
    q = torch.ones((1, 1, 1))
    bt = torch.tensor([[3, 1]], dtype=torch.int32)
    o = oracle_mod.decode(q, kc, vc, bt, torch.tensor([3], dtype=torch.int32), scale=1.0)
    e = math.e
    assert abs(float(o[0, 0, 0]) - e * e / (1 + e + e * e)) < 1e-15


def test_dominant_key_selects_its_value(oracle_mod):
    # One key aligned with q and scaled up: every other weight is at most exp(-gap).
    c, d, B = 20, 64, 16
    case = W.paged_case("dom", [c], 1, 1, d, B, torch.float32, 14)
    kc = case.k_cache.clone()
    t_star = 13
    phys = int(case.block_tables[0, t_star // B])
    kc[phys, 0, t_star % B] = case.q[0, 0] * 40.0
    o = oracle_mod.decode(case.q, kc, case.v_cache, case.block_tables, case.context_lens)
    v_star = case.v_cache[phys, 0, t_star % B].double()
    assert torch.allclose(o[0, 0], v_star, atol=1e-6, rtol=0)


def test_zero_length_gives_zero(oracle_mod):
    case = W.paged_case("z", [5, 0, 3], 2, 2, 64, 8, torch.float32, 15)
    o = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    assert torch.count_nonzero(o[1]) == 0
    assert torch.isfinite(o).all()


# ---- invariants of the definition --------------------------------------------------------------

def test_value_affine_map_commutes(oracle_mod):
    # The weights sum to 1, so o(aV + b) = a o(V) + b.  fp16 values make 2v + 0.5 exact in fp32.
    case = W.paged_case("aff", [33, 70], 4, 2, 64, 16, torch.float16, 16, sentinel="none")
    kc, vc = case.k_cache.float(), case.v_cache.float()
    o1 = oracle_mod.decode(case.q.float(), kc, vc, case.block_tables, case.context_lens)
    o2 = oracle_mod.decode(case.q.float(), kc, vc * 2 + 0.5, case.block_tables, case.context_lens)
    assert torch.allclose(o2, 2 * o1 + 0.5, atol=1e-12, rtol=0)


def test_output_inside_value_hull(oracle_mod):
    case = W.gqa8k_bf16(S=4)
    o = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, n_threads=4)
    B = case.B
    for s in range(case.S):
        c = int(case.context_lens[s])
        rows = [case.v_cache[int(case.block_tables[s, t // B]), :, t % B].double() for t in range(c)]
        V = torch.stack(rows)  # [c, Hk, d]
        lo, hi = V.min(0).values, V.max(0).values
        g = case.H // case.Hk
        for h in range(case.H):
            assert (o[s, h] >= lo[h // g] - 1e-12).all() and (o[s, h] <= hi[h // g] + 1e-12).all()


def test_score_shift_along_query_is_invisible(oracle_mod):
    # Adding the same multiple of q to every key adds one constant to every score of that head.
    # Small integers keep every stored value exact in fp32.
    g = torch.Generator().manual_seed(7)
    case = W.paged_case("shift", [45], 1, 1, 64, 16, torch.float32, 17, sentinel="none")
    q = torch.randint(-2, 3, case.q.shape, generator=g).float()
    kc = torch.randint(-8, 9, case.k_cache.shape, generator=g).float() / 4
    kc2 = kc + 0.25 * q[0, 0]
    o1 = oracle_mod.decode(q, kc, case.v_cache, case.block_tables, case.context_lens)
    o2 = oracle_mod.decode(q, kc2, case.v_cache, case.block_tables, case.context_lens)
    assert torch.allclose(o1, o2, atol=1e-12, rtol=0)


# ---- paging: identity table == contiguous attention (a library routine) --------------------------

@pytest.mark.parametrize("dtype,g,d,B", [(torch.float32, 1, 64, 16), (torch.float16, 4, 128, 8),
                                         (torch.bfloat16, 8, 128, 32), (torch.bfloat16, 2, 64, 16)])
def test_identity_table_equals_sdpa(oracle_mod, dtype, g, d, B):
    # "PagedAttention原理", 从虚拟内存的启发: blocks are logically contiguous though stored apart.
    # Store contiguous K/V in blocks 0, 1, 2, ... and compare with torch's fp64 attention.
    torch.manual_seed(0)
    Hk, S = 2, 3
    H = g * Hk
    lens = [1, B + 3, 3 * B]
    nbs = [(c + B - 1) // B for c in lens]
    n_blocks = sum(nbs)
    kc = torch.randn(n_blocks, Hk, B, d).to(dtype)
    vc = torch.randn(n_blocks, Hk, B, d).to(dtype)
    q = torch.randn(S, H, d).to(dtype)
    bt = torch.full((S, max(nbs)), -1, dtype=torch.int32)
    pos = 0
    for s in range(S):
        bt[s, : nbs[s]] = torch.arange(pos, pos + nbs[s], dtype=torch.int32)
        pos += nbs[s]
    o = oracle_mod.decode(q, kc, vc, bt, torch.tensor(lens, dtype=torch.int32))
    for s in range(S):
        blocks = bt[s, : nbs[s]].long()
        K = kc[blocks].permute(1, 0, 2, 3).reshape(Hk, -1, d)[:, : lens[s]].double()
        V = vc[blocks].permute(1, 0, 2, 3).reshape(Hk, -1, d)[:, : lens[s]].double()
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[s].double()[:, None, :], K, V, enable_gqa=True)[:, 0, :]
        assert torch.allclose(o[s], ref, atol=1e-12, rtol=1e-12)


# ---- physical placement does not matter --------------------------------------------------------

@pytest.mark.parametrize("B", [8, 16, 32])
def test_physical_permutation_is_bit_identical(oracle_mod, B):
    case = W.paged_case("perm", [1, B - 1, B, B + 1, 5 * B + 3], 8, 2, 64, B, torch.bfloat16, 18)
    o1 = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    n = case.n_blocks
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(5))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(n)
    kc2 = torch.empty_like(case.k_cache)
    vc2 = torch.empty_like(case.v_cache)
    kc2[perm] = case.k_cache
    vc2[perm] = case.v_cache
    bt2 = case.block_tables.clone()
    m = bt2 >= 0
    bt2[m] = perm[bt2[m].long()].to(torch.int32)
    o2 = oracle_mod.decode(case.q, kc2, vc2, bt2, case.context_lens)
    assert torch.equal(o1, o2)


def test_shared_prefix_sequences_match(oracle_mod):
    # "PagedAttention原理", 共享prompt: sequences sharing a prompt read the same physical blocks;
    # with identical tails and queries their outputs are identical.
    B, d, Hk, H = 16, 64, 2, 4
    case = W.paged_case("pref", [70, 70], H, Hk, d, B, torch.float16, 19, sentinel="none", n_blocks=20)
    bt = case.block_tables.clone()
    bt[1, :4] = bt[0, :4]          # share the four full prompt blocks
    kc, vc = case.k_cache.clone(), case.v_cache.clone()
    kc[int(bt[1, 4])] = kc[int(bt[0, 4])]   # identical tails stored in different blocks
    vc[int(bt[1, 4])] = vc[int(bt[0, 4])]
    q = case.q.clone()
    q[1] = q[0]
    o = oracle_mod.decode(q, kc, vc, bt, case.context_lens)
    assert torch.equal(o[0], o[1])


# ---- the block-wise formulation ("PagedAttention原理", 实现一个虚拟内存, eqs. A_ij, o_i) -----------------

@pytest.mark.parametrize("dtype,g,d,B", [(torch.float32, 1, 64, 16), (torch.float16, 4, 128, 8),
                                         (torch.bfloat16, 8, 128, 32), (torch.bfloat16, 4, 128, 16)])
def test_blockwise_formula_equals_gathered_softmax(oracle_mod, dtype, g, d, B):
    lens = [1, B - 1, B, B + 1, 3 * B + 5, 100]
    case = W.paged_case("bw", lens, 2 * g, 2, d, B, dtype, 20)
    o1 = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    o2 = oracle_mod.decode_blockwise(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    assert torch.allclose(o1, o2, atol=1e-12, rtol=1e-12)


@pytest.mark.parametrize("P", [16, 64, 96, 1000])
def test_partition_merge_equals_plain(oracle_mod, P):
    # The denominator of A_ij is a sum over blocks; splitting it over any set of partitions and
    # merging with max-rescaling gives the same o.
    lens = [1, 15, 16, 17, 200, 333]
    case = W.paged_case("pm", lens, 4, 2, 64, 16, torch.bfloat16, 21)
    n_parts = max((c + P - 1) // P for c in lens)
    po, pm, pl = oracle_mod.partials(case.q, case.k_cache, case.v_cache, case.block_tables,
                                     case.context_lens, P, n_parts)
    o1 = oracle_mod.combine(po, pm, pl)
    o0 = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    assert torch.allclose(o0, o1, atol=1e-12, rtol=1e-12)
    # each partial is itself the definition over its token range (single-part case)
    lens1 = torch.tensor([min(c, P) for c in lens], dtype=torch.int32)
    o_first = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, lens1)
    assert torch.allclose(po[:, :, 0] / pl[:, :, 0, None], o_first, atol=1e-12, rtol=1e-12)


def test_oracle_threads_do_not_change_results(oracle_mod):
    case = W.gqa8k_bf16(S=6)
    o1 = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, n_threads=1)
    o8 = oracle_mod.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, n_threads=8)
    assert torch.equal(o1, o8)


# ---- cache write and block copy (torch indexing as the independent routine) -----------------------

@pytest.mark.parametrize("dtype", DT)
def test_cache_write_matches_index_put(oracle_mod, dtype):
    n_blocks, Hk, B, d, T = 10, 3, 8, 64, 12
    g = torch.Generator().manual_seed(3)
    kc = torch.randn(n_blocks, Hk, B, d, generator=g).to(dtype)
    vc = torch.randn(n_blocks, Hk, B, d, generator=g).to(dtype)
    key = torch.randn(T, Hk, d, generator=g).to(dtype)
    val = torch.randn(T, Hk, d, generator=g).to(dtype)
    slots = torch.randperm(n_blocks * B, generator=g)[:T].to(torch.int64)
    slots[3] = -1  # padding token
    k2, v2 = oracle_mod.cache_write(kc, vc, key, val, slots)
    kr = kc.clone().permute(0, 2, 1, 3).reshape(n_blocks * B, Hk, d)
    vr = vc.clone().permute(0, 2, 1, 3).reshape(n_blocks * B, Hk, d)
    keep = slots >= 0
    kr[slots[keep]] = key[keep]
    vr[slots[keep]] = val[keep]
    kr = kr.reshape(n_blocks, B, Hk, d).permute(0, 2, 1, 3)
    vr = vr.reshape(n_blocks, B, Hk, d).permute(0, 2, 1, 3)
    assert torch.equal(k2, kr.contiguous()) and torch.equal(v2, vr.contiguous())


@pytest.mark.parametrize("dtype", DT)
def test_copy_blocks_matches_index_copy(oracle_mod, dtype):
    n_blocks, Hk, B, d = 12, 2, 16, 64
    g = torch.Generator().manual_seed(4)
    kc = torch.randn(n_blocks, Hk, B, d, generator=g).to(dtype)
    vc = torch.randn(n_blocks, Hk, B, d, generator=g).to(dtype)
    pairs = torch.tensor([[1, 7], [3, 9], [1, 11]], dtype=torch.int32)
    k2, v2 = oracle_mod.copy_blocks(kc, vc, pairs)
    kr, vr = kc.clone(), vc.clone()
    kr[pairs[:, 1].long()] = kc[pairs[:, 0].long()]
    vr[pairs[:, 1].long()] = vc[pairs[:, 0].long()]
    assert torch.equal(k2, kr) and torch.equal(v2, vr)
    # the source blocks are untouched ("解决COW": the shared block stays as it was)
    assert torch.equal(k2[1], kc[1]) and torch.equal(k2[3], kc[3])


@pytest.mark.parametrize("dtype", DT)
def test_swap_blocks_matches_index_copy(oracle_mod, dtype):
    # "PagedAttention原理", 抢占与恢复 (swap): blocks move between the GPU pool and a CPU pool.
    Hk, B, d = 2, 8, 64
    g = torch.Generator().manual_seed(5)
    dev_k = torch.randn(10, Hk, B, d, generator=g).to(dtype)
    dev_v = torch.randn(10, Hk, B, d, generator=g).to(dtype)
    host_k = torch.randn(6, Hk, B, d, generator=g).to(dtype)
    host_v = torch.randn(6, Hk, B, d, generator=g).to(dtype)
    out_pairs = torch.tensor([[7, 0], [2, 5], [9, 3]], dtype=torch.int32)   # device -> host
    hk, hv = oracle_mod.swap_blocks(host_k, host_v, dev_k, dev_v, out_pairs)
    rk, rv = host_k.clone(), host_v.clone()
    rk[out_pairs[:, 1].long()] = dev_k[out_pairs[:, 0].long()]
    rv[out_pairs[:, 1].long()] = dev_v[out_pairs[:, 0].long()]
    assert torch.equal(hk, rk) and torch.equal(hv, rv)
    in_pairs = torch.tensor([[0, 1], [5, 4], [3, 8]], dtype=torch.int32)    # host -> device, new ids
    dk, dv = oracle_mod.swap_blocks(dev_k, dev_v, hk, hv, in_pairs)
    assert torch.equal(dk[1], dev_k[7]) and torch.equal(dk[4], dev_k[2]) and torch.equal(dv[8], dev_v[9])
    with pytest.raises(ValueError):
        oracle_mod.swap_blocks(dev_k, dev_v, hk, hv, torch.tensor([[6, 0]], dtype=torch.int32))


# ---- prefill / mixed batches (causal, several query tokens per sequence) ----------------------------

@pytest.mark.parametrize("dtype,g,d,B", [(torch.float32, 1, 64, 16), (torch.bfloat16, 4, 128, 16),
                                         (torch.float16, 8, 128, 8)])
def test_prefill_identity_table_equals_causal_sdpa(oracle_mod, dtype, g, d, B):
    # Contiguous blocks, the whole context as the query chunk: causal attention over the prompt.
    torch.manual_seed(1)
    Hk, H = 2, 2 * g
    lens = [1, 7, B + 5, 3 * B]
    nbs = [(c + B - 1) // B for c in lens]
    kc = torch.randn(sum(nbs), Hk, B, d).to(dtype)
    vc = torch.randn(sum(nbs), Hk, B, d).to(dtype)
    bt = torch.full((len(lens), max(nbs)), -1, dtype=torch.int32)
    pos = 0
    for s, nb in enumerate(nbs):
        bt[s, :nb] = torch.arange(pos, pos + nb, dtype=torch.int32)
        pos += nb
    q_start = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32)
    q = torch.randn(int(q_start[-1]), H, d).to(dtype)
    o = oracle_mod.prefill(q, q_start, kc, vc, bt, torch.tensor(lens, dtype=torch.int32))
    for s, c in enumerate(lens):
        blocks = bt[s, : nbs[s]].long()
        K = kc[blocks].permute(1, 0, 2, 3).reshape(Hk, -1, d)[:, :c].double()
        V = vc[blocks].permute(1, 0, 2, 3).reshape(Hk, -1, d)[:, :c].double()
        qs = q[q_start[s]: q_start[s + 1]].double().permute(1, 0, 2)        # [H, c, d]
        ref = torch.nn.functional.scaled_dot_product_attention(qs, K, V, is_causal=True, enable_gqa=True)
        assert torch.allclose(o[q_start[s]: q_start[s + 1]], ref.permute(1, 0, 2), atol=1e-12, rtol=1e-12)


def test_prefill_single_token_equals_decode(oracle_mod):
    # Decode is the n_s = 1 case: a mixed batch of decode rows and prefill chunks must agree with
    # the decode definition on its decode rows, and on each chunk's last row.
    case = W.paged_case("mix", [40, 130, 1, 77], 8, 2, 64, 16, torch.bfloat16, 22)
    n = [1, 17, 1, 5]
    q_start = torch.tensor([0] + list(torch.tensor(n).cumsum(0)), dtype=torch.int32)
    g = torch.Generator().manual_seed(3)
    q = torch.randn(int(q_start[-1]), 8, 64, generator=g).to(torch.bfloat16)
    o = oracle_mod.prefill(q, q_start, case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    last_rows = (q_start[1:] - 1).long()
    od = oracle_mod.decode(q[last_rows], case.k_cache, case.v_cache, case.block_tables, case.context_lens)
    assert torch.allclose(o[last_rows], od, atol=1e-13, rtol=0)
    # an earlier chunk row equals decode with the context cut at its position
    lens2 = case.context_lens.clone()
    lens2[1] = 130 - 17 + 3 + 1
    od2 = oracle_mod.decode(q[q_start[1] + 3: q_start[1] + 4].expand(4, -1, -1).contiguous(), case.k_cache,
                            case.v_cache, case.block_tables, lens2)
    assert torch.allclose(o[q_start[1] + 3], od2[1], atol=1e-13, rtol=0)


def _brute_layout(rnd, lens, Hk, d, B):
    """A tiny paged cache in plain Python: blocks at shuffled physical ids, fp32-exact values."""
    nb = [-(-c // B) for c in lens]
    n_blocks = sum(nb) + 2
    phys = list(range(n_blocks))
    rnd.shuffle(phys)
    kc = torch.full((n_blocks, Hk, B, d), float("nan"))
    vc = torch.full((n_blocks, Hk, B, d), float("nan"))
    tables = torch.full((len(lens), max(max(nb), 1)), -1, dtype=torch.int32)
    i = 0
    for s, c in enumerate(lens):
        for j in range(nb[s]):
            tables[s, j] = phys[i]
            i += 1
        for t in range(c):
            p = int(tables[s, t // B])
            for kh in range(Hk):
                for e in range(d):
                    kc[p, kh, t % B, e] = rnd.randint(-8, 8) / 4.0
                    vc[p, kh, t % B, e] = rnd.randint(-8, 8) / 4.0
    return kc, vc, tables


def _brute_attend(qv, kc, vc, table, kh, n_keys, B, scale):
    xs = []
    for t in range(n_keys):
        p, o = int(table[t // B]), t % B
        xs.append(scale * sum(float(qv[e]) * float(kc[p, kh, o, e]) for e in range(len(qv))))
    m = max(xs)
    w = [math.exp(x - m) for x in xs]
    z = sum(w)
    return [sum(w[t] * float(vc[int(table[t // B]), kh, t % B, e]) for t in range(n_keys)) / z
            for e in range(len(qv))]


def test_brute_force_tiny_decode(oracle_mod):
    # every (d <= 4, c <= 5, B in {1, 2}, g in {1, 2}) shape class, expanded by plain Python loops
    rnd = random.Random(2024)
    for trial in range(40):
        d, B, g, Hk = rnd.randint(1, 4), rnd.choice([1, 2]), rnd.choice([1, 2]), rnd.choice([1, 2])
        lens = [rnd.randint(1, 5) for _ in range(rnd.randint(1, 3))]
        kc, vc, tables = _brute_layout(rnd, lens, Hk, d, B)
        H = Hk * g
        q = torch.tensor([[[rnd.randint(-8, 8) / 4.0 for _ in range(d)] for _ in range(H)] for _ in lens])
        scale = rnd.choice([1.0, 0.5, 0.7])
        o = oracle_mod.decode(q, kc, vc, tables, torch.tensor(lens, dtype=torch.int32), scale=scale)
        for s, c in enumerate(lens):
            for h in range(H):
                ref = _brute_attend(q[s, h].tolist(), kc, vc, tables[s], h // g, c, B, scale)
                for e in range(d):
                    assert abs(float(o[s, h, e]) - ref[e]) <= 1e-12 * (1 + abs(ref[e])), (trial, s, h, e)


def test_brute_force_tiny_prefill(oracle_mod):
    # the token at position p = c - n + i attends to keys 0 .. p (plain Python loops)
    rnd = random.Random(2025)
    for trial in range(30):
        d, B, g, Hk = rnd.randint(1, 4), rnd.choice([1, 2]), rnd.choice([1, 2]), 1
        lens = [rnd.randint(1, 5) for _ in range(rnd.randint(1, 3))]
        nq = [rnd.randint(0, c) for c in lens]
        kc, vc, tables = _brute_layout(rnd, lens, Hk, d, B)
        H = Hk * g
        T = sum(nq)
        q = torch.tensor([[[rnd.randint(-8, 8) / 4.0 for _ in range(d)] for _ in range(H)] for _ in range(T)])
        q_start = torch.tensor([0] + [sum(nq[:i + 1]) for i in range(len(nq))], dtype=torch.int32)
        o = oracle_mod.prefill(q.reshape(T, H, d), q_start, kc, vc, tables, torch.tensor(lens, dtype=torch.int32),
                               scale=1.0)
        for s, c in enumerate(lens):
            for i in range(nq[s]):
                row, pos = int(q_start[s]) + i, c - nq[s] + i
                for h in range(H):
                    ref = _brute_attend(q[row, h].tolist(), kc, vc, tables[s], h // g, pos + 1, B, 1.0)
                    for e in range(d):
                        assert abs(float(o[row, h, e]) - ref[e]) <= 1e-12 * (1 + abs(ref[e])), (trial, s, i, h)
