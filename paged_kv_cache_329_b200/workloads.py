"""Seeded synthetic inputs for paged decode attention.

This module only draws random numbers and lays them out; it holds none of the attention,
cache-write, copy or block-manager arithmetic.  It is the one piece of code that feeds both the
CUDA path and the oracle, so both always see identical inputs.

The five serving scenarios (shapes from the pages' discussion of decode serving: variable
context lengths, block sizes 8/16/32 with 16 the common default, parallel sampling and beam
search sharing a prompt's blocks, long contexts):

  tiny_fp32        4 seqs, 8/8 heads, d=64,  B=16, c ~ U{1..200}, pool of 64 blocks, fp32
  mha13b_fp16      64 seqs, 40/40 heads, d=128, B=16, c ~ U{1..2048}, pool 1.25x, fp16,
                   plus one new token per sequence written through a slot mapping
  gqa8k_bf16       256 seqs, 32/8 heads, d=128, B=16, c = clip(round(exp(ln 1024 + N(0,1))), 16, 8192)
  shared_prefix    32 requests x 4 seqs, 32/8 heads, d=128, B=16, 1024-token prompt, tails U{0..256}
  long_bf16        16 seqs, 64/8 heads, d=128, B in {8,16,32}, c ~ U{16384..32768}

Random values are drawn as float32 N(0,1) from a seeded torch.Generator and cast to the cache
type with round-to-nearest-even.  Physical blocks are handed to sequences, in logical order, from
a seeded random permutation of the pool, so logically adjacent blocks are scattered in memory.
Unused pool blocks and the unused slots of partly filled last blocks hold NaN when
``sentinel="nan"``: a kernel that reads a token it should not read then produces NaN.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass
class DecodeCase:
    name: str
    q: torch.Tensor             # [S, H, d]
    k_cache: torch.Tensor       # [n_blocks, Hk, B, d]
    v_cache: torch.Tensor       # [n_blocks, Hk, B, d]
    block_tables: torch.Tensor  # [S, max_blocks_per_seq] int32, padding -1
    context_lens: torch.Tensor  # [S] int32
    scale: float
    H: int
    Hk: int
    d: int
    B: int

    @property
    def S(self) -> int:
        return self.q.shape[0]

    @property
    def n_blocks(self) -> int:
        return self.k_cache.shape[0]

    def to(self, device) -> "DecodeCase":
        f = lambda t: t.to(device)
        return DecodeCase(self.name, f(self.q), f(self.k_cache), f(self.v_cache), f(self.block_tables),
                          f(self.context_lens), self.scale, self.H, self.Hk, self.d, self.B)


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn(gen: torch.Generator, shape, dtype, device="cpu") -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32, device=device).to(dtype)


# ---- context-length distributions --------------------------------------------------------------

def lens_uniform(gen, S, lo, hi):
    return torch.randint(lo, hi + 1, (S,), generator=gen, dtype=torch.int64)


def lens_lognormal(gen, S, median, sigma, lo, hi):
    z = torch.randn((S,), generator=gen, dtype=torch.float64)
    c = torch.exp(math.log(median) + sigma * z).round()
    return c.clamp(lo, hi).to(torch.int64)


# ---- paged layout -------------------------------------------------------------------------------

def paged_case(name, lens, H, Hk, d, B, dtype, seed, *, pool_factor=1.25, n_blocks=None,
               sentinel="nan", device="cpu", extra_blocks_per_seq=0) -> DecodeCase:
    """Random q/K/V for the given context lengths, stored in a shuffled block pool."""
    gen = generator(seed)
    lens = torch.as_tensor(lens, dtype=torch.int64)
    S = lens.numel()
    nb = [(int(c) + B - 1) // B for c in lens]
    need = sum(nb)
    if n_blocks is None:
        n_blocks = max(1, math.ceil(pool_factor * need))
    if n_blocks < need:
        raise ValueError("pool smaller than the blocks needed")
    perm = torch.randperm(n_blocks, generator=gen)
    max_nb = max(1, max(nb) + extra_blocks_per_seq)
    tables = torch.full((S, max_nb), -1, dtype=torch.int32)
    pos = 0
    for s in range(S):
        tables[s, : nb[s]] = perm[pos: pos + nb[s]].to(torch.int32)
        pos += nb[s]
    q = randn(gen, (S, H, d), dtype)
    dev_gen = generator(seed + 1000, device) if torch.device(device).type == "cuda" else gen
    k = randn(dev_gen, (n_blocks, Hk, B, d), dtype, device)
    v = randn(dev_gen, (n_blocks, Hk, B, d), dtype, device)
    if sentinel == "nan":
        used = torch.zeros((n_blocks, B), dtype=torch.bool)
        for s in range(S):
            c = int(lens[s])
            for j in range(nb[s]):
                filled = min(B, c - j * B)
                used[int(tables[s, j]), :filled] = True
        mask = (~used).to(k.device)[:, None, :, None].expand_as(k)
        k = k.masked_fill(mask, float("nan"))
        v = v.masked_fill(mask, float("nan"))
    return DecodeCase(name, q.to(device), k, v, tables.to(device), lens.to(torch.int32).to(device),
                      1.0 / math.sqrt(d), H, Hk, d, B)


# ---- the scenarios ------------------------------------------------------------------------------

def tiny_fp32(sentinel="nan", device="cpu"):
    gen = generator(1)
    lens = lens_uniform(gen, 4, 1, 200)
    return paged_case("tiny_fp32", lens, 8, 8, 64, 16, torch.float32, 1, n_blocks=64,
                      sentinel=sentinel, device=device)


def mha13b_fp16(sentinel="nan", device="cpu"):
    gen = generator(2)
    lens = lens_uniform(gen, 64, 1, 2048)
    return paged_case("mha13b_fp16", lens, 40, 40, 128, 16, torch.float16, 2, sentinel=sentinel, device=device)


def gqa8k_lens(S=256):
    return lens_lognormal(generator(3), S, 1024.0, 1.0, 16, 8192)


def gqa8k_bf16(sentinel="nan", device="cpu", S=256):
    return paged_case("gqa8k_bf16", gqa8k_lens(S), 32, 8, 128, 16, torch.bfloat16, 3,
                      sentinel=sentinel, device=device)


def long_bf16(B=16, sentinel="nan", device="cpu", S=16):
    gen = generator(5)
    lens = lens_uniform(gen, S, 16384, 32768)
    return paged_case(f"long_bf16_B{B}", lens, 64, 8, 128, B, torch.bfloat16, 5,
                      sentinel=sentinel, device=device)


def new_token_slots(case: DecodeCase, gen: torch.Generator):
    """One new token per sequence: its slot is position c_s of the sequence (a fresh block from
    the unused part of the pool when the last block is full).  Returns the grown block tables,
    the grown lengths and the slot mapping [S] int64; distinct sequences get distinct slots."""
    tables = case.block_tables.cpu().clone()
    lens = case.context_lens.cpu().to(torch.int64).clone()
    B = case.B
    used = set(int(x) for x in tables.flatten().tolist() if x >= 0)
    free = [b for b in torch.randperm(case.n_blocks, generator=gen).tolist() if b not in used]
    need_cols = int(((lens + 1 + B - 1) // B).max())
    if need_cols > tables.shape[1]:
        tables = torch.cat([tables, torch.full((tables.shape[0], need_cols - tables.shape[1]), -1,
                                               dtype=torch.int32)], 1)
    slots = torch.empty(case.S, dtype=torch.int64)
    for s in range(case.S):
        c = int(lens[s])
        j, off = divmod(c, B)
        if off == 0:
            tables[s, j] = free.pop()
        slots[s] = int(tables[s, j]) * B + off
        lens[s] = c + 1
    return tables, lens.to(torch.int32), slots


CONFIGS = {
    "tiny_fp32": dict(S=4, H=8, Hk=8, d=64, B=16, dtype="f32"),
    "mha13b_fp16": dict(S=64, H=40, Hk=40, d=128, B=16, dtype="f16"),
    "gqa8k_bf16": dict(S=256, H=32, Hk=8, d=128, B=16, dtype="bf16"),
    "shared_prefix_bf16": dict(S=128, H=32, Hk=8, d=128, B=16, dtype="bf16"),
    "long_bf16": dict(S=16, H=64, Hk=8, d=128, B=16, dtype="bf16"),
}
