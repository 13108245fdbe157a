"""Oracle: plain fp64 CPU restatements of paged decode attention and its companion paths.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The product library never loads it, and it shares
no code with the CUDA path: ``oracle.cpp`` re-derives element decoding, indexing and the
attention arithmetic from the pages, and ``allocator.py`` restates the block-manager rules.

Functions take torch CPU tensors (any of float32 / float16 / bfloat16 for the floating inputs,
int32 block tables and lengths, int64 slot mappings) and return float64 tensors.

Pages followed (title, section, equation):
  * "PagedAttention原理", "为什么会有 KV cache": o_t = softmax(q_t K^T / sqrt(d)) V  -> decode()
  * "PagedAttention原理", "实现一个虚拟内存": K_j, V_j, A_ij, o_i              -> decode_blockwise(),
    partials(), combine()
  * "vllm" (cnblogs), 2.2 Decode: the new token's K,V are stored in the cache -> cache_write()
  * "PagedAttention原理", "解决COW", step 2 (copy the shared block)        -> copy_blocks()
  * "PagedAttention原理", "抢占与恢复", swap (blocks to CPU memory and back)  -> swap_blocks()
  * Orca notes (selective batching) and "vllm" 2.1 Prefill: several causal query tokens per
    sequence, decode being one                                                -> prefill()
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}


def build(force: bool = False) -> str:
    """Compile ``oracle.cpp`` into ``liboracle.so`` with g++ (no GPU code involved)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _declare(lib):
    P, I, D, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_long
    lib.oracle_decode.argtypes = [P, P, I, P, P, I, P, P, I, I, I, I, I, I, I, D, I]
    lib.oracle_decode.restype = I
    lib.oracle_decode_blockwise.argtypes = [P, P, I, P, P, I, P, P, I, I, I, I, I, I, I, D]
    lib.oracle_decode_blockwise.restype = I
    lib.oracle_partials.argtypes = [P, P, P, I, I, P, I, P, P, I, P, P, I, I, I, I, I, I, I, D]
    lib.oracle_partials.restype = I
    lib.oracle_combine.argtypes = [P, P, P, P, I, I, I, I, I]
    lib.oracle_combine.restype = None
    lib.oracle_cache_write.argtypes = [P, P, P, P, P, I, I, I, I, I, I]
    lib.oracle_cache_write.restype = I
    lib.oracle_copy_blocks.argtypes = [P, P, P, I, I, I, I, I, I]
    lib.oracle_copy_blocks.restype = I
    lib.oracle_prefill.argtypes = [P, P, I, P, P, P, I, P, P, I, I, I, I, I, I, I, D, I]
    lib.oracle_prefill.restype = I
    lib.oracle_swap_blocks.argtypes = [P, P, I, P, P, I, P, I, I, I, I, I]
    lib.oracle_swap_blocks.restype = I
    lib.oracle_hardware_threads.argtypes = []
    lib.oracle_hardware_threads.restype = I
    lib.oracle_elem_to_double.argtypes = [P, I, L]
    lib.oracle_elem_to_double.restype = D
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


_active = None  # a library other than liboracle.so while `variant(...)` is in effect


def _L():
    return _active if _active is not None else _load()


class variant:
    """Context manager: route every function of this module to another build of oracle.cpp
    (used by the tests that check the pins catch planted mistakes)."""

    def __init__(self, so_path: str):
        self.lib = _declare(ctypes.CDLL(so_path))

    def __enter__(self):
        global _active
        self._prev, _active = _active, self.lib
        return self

    def __exit__(self, *exc):
        global _active
        _active = self._prev
        return False


def _cpu(t: torch.Tensor) -> torch.Tensor:
    if t.device.type != "cpu":
        raise ValueError("the oracle takes CPU tensors only")
    return t.contiguous()


def _code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPE_CODE:
        raise ValueError(f"unsupported element type {t.dtype}")
    return _DTYPE_CODE[t.dtype]


def hardware_threads() -> int:
    return _L().oracle_hardware_threads()


def elem_to_double(t: torch.Tensor, idx: int) -> float:
    t = _cpu(t)
    return _L().oracle_elem_to_double(t.data_ptr(), _code(t), idx)


def _shape(q, k_cache, block_tables):
    S, H, d = q.shape
    n_blocks, Hk, B, d2 = k_cache.shape
    if d2 != d:
        raise ValueError("head_dim mismatch")
    return S, H, d, n_blocks, Hk, B, block_tables.shape[1]


def decode(q, k_cache, v_cache, block_tables, context_lens, scale=None, n_threads=1):
    """softmax(scale * q K^T) V per (sequence, query head) over the gathered cache; [S, H, d] fp64."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    bt, cl = _cpu(block_tables.to(torch.int32)), _cpu(context_lens.to(torch.int32))
    S, H, d, n_blocks, Hk, B, mb = _shape(q, k_cache, bt)
    if scale is None:
        scale = 1.0 / d ** 0.5
    out = torch.empty((S, H, d), dtype=torch.float64)
    rc = _L().oracle_decode(
        out.data_ptr(), q.data_ptr(), _code(q), k_cache.data_ptr(), v_cache.data_ptr(), _code(k_cache),
        bt.data_ptr(), cl.data_ptr(), S, H, Hk, d, B, n_blocks, mb, float(scale), int(n_threads),
    )
    if rc != 0:
        raise ValueError(f"oracle_decode failed ({rc}): block table entry out of range")
    return out


def decode_blockwise(q, k_cache, v_cache, block_tables, context_lens, scale=None):
    """The block-wise A_ij / o_i formulation, literally (no max subtraction); [S, H, d] fp64."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    bt, cl = _cpu(block_tables.to(torch.int32)), _cpu(context_lens.to(torch.int32))
    S, H, d, n_blocks, Hk, B, mb = _shape(q, k_cache, bt)
    if scale is None:
        scale = 1.0 / d ** 0.5
    out = torch.empty((S, H, d), dtype=torch.float64)
    rc = _L().oracle_decode_blockwise(
        out.data_ptr(), q.data_ptr(), _code(q), k_cache.data_ptr(), v_cache.data_ptr(), _code(k_cache),
        bt.data_ptr(), cl.data_ptr(), S, H, Hk, d, B, n_blocks, mb, float(scale),
    )
    if rc != 0:
        raise ValueError(f"oracle_decode_blockwise failed ({rc})")
    return out


def partials(q, k_cache, v_cache, block_tables, context_lens, partition_size, n_parts, scale=None):
    """Per-partition (o~, m, l) states; part p covers tokens [p*P, min((p+1)*P, c))."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    bt, cl = _cpu(block_tables.to(torch.int32)), _cpu(context_lens.to(torch.int32))
    S, H, d, n_blocks, Hk, B, mb = _shape(q, k_cache, bt)
    if scale is None:
        scale = 1.0 / d ** 0.5
    po = torch.empty((S, H, n_parts, d), dtype=torch.float64)
    pm = torch.empty((S, H, n_parts), dtype=torch.float64)
    pl = torch.empty((S, H, n_parts), dtype=torch.float64)
    rc = _L().oracle_partials(
        po.data_ptr(), pm.data_ptr(), pl.data_ptr(), n_parts, partition_size, q.data_ptr(), _code(q),
        k_cache.data_ptr(), v_cache.data_ptr(), _code(k_cache), bt.data_ptr(), cl.data_ptr(),
        S, H, Hk, d, B, n_blocks, mb, float(scale),
    )
    if rc != 0:
        raise ValueError(f"oracle_partials failed ({rc})")
    return po, pm, pl


def combine(part_o, part_m, part_l):
    """Merge per-partition states into o; inputs fp32 or fp64 [S,H,P,d] / [S,H,P]."""
    S, H, n_parts, d = part_o.shape
    f32 = part_o.dtype == torch.float32
    want = torch.float32 if f32 else torch.float64
    po, pm, pl = (_cpu(t.to(want)) for t in (part_o, part_m, part_l))
    out = torch.empty((S, H, d), dtype=torch.float64)
    _L().oracle_combine(out.data_ptr(), po.data_ptr(), pm.data_ptr(), pl.data_ptr(), int(f32), S, H, n_parts, d)
    return out


def cache_write(k_cache, v_cache, key, value, slot_mapping):
    """Slot-mapped write into copies of the caches; returns (k_cache', v_cache')."""
    kc, vc = _cpu(k_cache).clone(), _cpu(v_cache).clone()
    key, value = _cpu(key.to(kc.dtype)), _cpu(value.to(kc.dtype))
    sm = _cpu(slot_mapping.to(torch.int64))
    n_blocks, Hk, B, d = kc.shape
    rc = _L().oracle_cache_write(
        kc.data_ptr(), vc.data_ptr(), key.data_ptr(), value.data_ptr(), sm.data_ptr(),
        key.shape[0], Hk, d, B, n_blocks, _code(kc),
    )
    if rc != 0:
        raise ValueError("oracle_cache_write: slot out of range")
    return kc, vc


def copy_blocks(k_cache, v_cache, pairs):
    """Whole-block copies src -> dst in copies of the caches; returns (k_cache', v_cache')."""
    kc, vc = _cpu(k_cache).clone(), _cpu(v_cache).clone()
    pr = _cpu(pairs.to(torch.int32).reshape(-1, 2))
    n_blocks, Hk, B, d = kc.shape
    rc = _L().oracle_copy_blocks(kc.data_ptr(), vc.data_ptr(), pr.data_ptr(), pr.shape[0], Hk, d, B, n_blocks, _code(kc))
    if rc != 0:
        raise ValueError("oracle_copy_blocks: block id out of range")
    return kc, vc


def swap_blocks(dst_k, dst_v, src_k, src_v, pairs):
    """Whole-block copies from a source pool into copies of a destination pool; returns (dst_k', dst_v')."""
    dk, dv = _cpu(dst_k).clone(), _cpu(dst_v).clone()
    sk, sv = _cpu(src_k), _cpu(src_v)
    pr = _cpu(pairs.to(torch.int32).reshape(-1, 2))
    n_dst, Hk, B, d = dk.shape
    if sk.shape[1:] != dk.shape[1:] or sk.dtype != dk.dtype:
        raise ValueError("pools must share the block layout and type")
    rc = _L().oracle_swap_blocks(dk.data_ptr(), dv.data_ptr(), n_dst, sk.data_ptr(), sv.data_ptr(), sk.shape[0],
                                 pr.data_ptr(), pr.shape[0], Hk, d, B, _code(dk))
    if rc != 0:
        raise ValueError("oracle_swap_blocks: block id out of range")
    return dk, dv


def prefill(q, q_start, k_cache, v_cache, block_tables, context_lens, scale=None, n_threads=1):
    """Causal attention of each sequence's last n_s tokens over its paged context; [T, H, d] fp64."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    qs = _cpu(q_start.to(torch.int32))
    bt, cl = _cpu(block_tables.to(torch.int32)), _cpu(context_lens.to(torch.int32))
    T, H, d = q.shape
    n_blocks, Hk, B, d2 = k_cache.shape
    S = cl.numel()
    if scale is None:
        scale = 1.0 / d ** 0.5
    out = torch.empty((T, H, d), dtype=torch.float64)
    rc = _L().oracle_prefill(out.data_ptr(), q.data_ptr(), _code(q), qs.data_ptr(), k_cache.data_ptr(),
                             v_cache.data_ptr(), _code(k_cache), bt.data_ptr(), cl.data_ptr(), S, H, Hk, d, B,
                             n_blocks, bt.shape[1], float(scale), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_prefill failed ({rc})")
    return out
