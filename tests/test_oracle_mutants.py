"""The pins catch planted mistakes: each test builds a copy of oracle.cpp with one plausible error
(a dropped term, a wrong sign, index or operand) on the CPU and checks that at least one pin of
test_oracle_pins fails on it, while the unaltered oracle passes them all."""
import os
import subprocess
import tempfile

import pytest
import torch

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.cpp")

# (name, text in oracle.cpp, replacement); every occurrence is replaced
MUTANTS = [
    ("gqa head mapping", "h / g", "h % Hk"),
    ("offset inside a block", "* B + (t % B);", "* B + ((t + 1) % B);"),
    ("scale dropped", "x[t] = scale * acc;", "x[t] = acc;"),
    ("softmax sign", "x[t] = std::exp(x[t] - mx);", "x[t] = std::exp(mx - x[t]);"),
    ("normalisation dropped", "for (int i = 0; i < d; ++i) o[i] /= z;", "for (int i = 0; i < d; ++i) o[i] /= 1.0;"),
    ("values read from the key cache", "V[static_cast<size_t>(t) * d + i] = load_elem(v_cache",
     "V[static_cast<size_t>(t) * d + i] = load_elem(k_cache"),
    ("last token dropped", "    const int c = context_lens[s];\n    for (int i = 0; i < d; ++i) o[i] = 0.0;",
     "    const int c = context_lens[s] - (context_lens[s] > 1 ? 1 : 0);\n    for (int i = 0; i < d; ++i) o[i] = 0.0;"),
    ("transposed key operand", "acc += qv[i] * K[static_cast<size_t>(t) * d + i];",
     "acc += qv[i] * K[static_cast<size_t>(i) * c + t];"),
    ("bf16 widening", "static_cast<uint32_t>(b) << 16;", "static_cast<uint32_t>(b) << 15;"),
    ("fp16 exponent bias", "expo - 25", "expo - 24"),
    ("block-wise: last block unmasked", "const int filled = (j == nb - 1) ? c - j * B : B;", "const int filled = B;"),
    ("combine: sum weight dropped", "den += w * rd(part_l, base + p);", "den += rd(part_l, base + p);"),
    ("partials: values from keys", "o[i] += w * load_elem(v_cache, kv_dtype, rows[t - t0] * d + i);",
     "o[i] += w * load_elem(k_cache, kv_dtype, rows[t - t0] * d + i);"),
    ("cache write: block and offset swapped", "const int64_t blk = slot / B, off = slot % B;",
     "const int64_t blk = slot % B, off = slot / B;"),
    ("prefill: causal limit off by one (no self-attention)", "t <= pos", "t < pos"),
    ("prefill: query position taken from the chunk start", "const int pos = c - n + (row - q_start[s]);",
     "const int pos = c - n;"),
    ("swap: source and destination pools swapped",
     "std::memcpy(static_cast<char*>(dst_k) + dst * bytes, static_cast<const char*>(src_k) + src * bytes, bytes);",
     "std::memcpy(static_cast<char*>(dst_k) + dst * bytes, static_cast<const char*>(src_k) + dst * bytes, bytes);"),
    ("copy: value cache not copied",
     "std::memcpy(static_cast<char*>(v_cache) + dst * bytes, static_cast<const char*>(v_cache) + src * bytes, bytes);",
     "(void)0;"),
]

PINS = [
    lambda o: pins.test_elem_decoding_matches_torch(o, torch.float16),
    lambda o: pins.test_elem_decoding_matches_torch(o, torch.bfloat16),
    lambda o: pins.test_single_token_returns_its_value(o, torch.bfloat16),
    lambda o: pins.test_equal_keys_give_mean_of_values(o),
    lambda o: pins.test_three_token_closed_form(o),
    lambda o: pins.test_identity_table_equals_sdpa(o, torch.float32, 1, 64, 16),
    lambda o: pins.test_identity_table_equals_sdpa(o, torch.float16, 4, 128, 8),
    lambda o: pins.test_physical_permutation_is_bit_identical(o, 16),
    lambda o: pins.test_blockwise_formula_equals_gathered_softmax(o, torch.bfloat16, 4, 128, 16),
    lambda o: pins.test_partition_merge_equals_plain(o, 96),
    lambda o: pins.test_cache_write_matches_index_put(o, torch.bfloat16),
    lambda o: pins.test_copy_blocks_matches_index_copy(o, torch.bfloat16),
    lambda o: pins.test_swap_blocks_matches_index_copy(o, torch.bfloat16),
    lambda o: pins.test_prefill_identity_table_equals_causal_sdpa(o, torch.bfloat16, 4, 128, 16),
    lambda o: pins.test_prefill_single_token_equals_decode(o),
    lambda o: pins.test_brute_force_tiny_decode(o),
    lambda o: pins.test_brute_force_tiny_prefill(o),
]


def _failures(mod):
    n = 0
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, RuntimeError, IndexError):
            n += 1
    return n


@pytest.fixture(scope="module")
def tmpdir_mutants():
    with tempfile.TemporaryDirectory() as d:
        yield d


def test_unaltered_oracle_passes_the_pins(oracle_mod):
    assert _failures(oracle_mod) == 0


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(oracle_mod, tmpdir_mutants, name, old, new):
    src = open(SRC).read()
    assert old in src, f"mutation site for '{name}' not found"
    path = os.path.join(tmpdir_mutants, f"m{MUTANTS.index((name, old, new))}")
    open(path + ".cpp", "w").write(src.replace(old, new))
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-pthread", "-o", path + ".so",
                           path + ".cpp"])
    with oracle.variant(path + ".so"):
        assert _failures(oracle) >= 1, f"no pin caught the mutant '{name}'"
