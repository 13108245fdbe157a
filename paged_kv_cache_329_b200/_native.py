"""ctypes loader for libpa.so: declares every C entry point of include/pa.h.

The library is built in-tree (``python -m paged_kv_cache_329_b200.build``).  There is no fallback:
if libpa.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
SZ = ctypes.c_size_t
I32P = ctypes.POINTER(ctypes.c_int32)
I64P = ctypes.POINTER(ctypes.c_int64)
IP = ctypes.POINTER(ctypes.c_int)

class StepDesc(ctypes.Structure):
    """pa_step_desc of include/pa.h, field for field."""
    _fields_ = [
        ("h_query", P), ("h_key", P), ("h_value", P), ("h_slots", P), ("h_pairs", P), ("h_n_pairs", P),
        ("h_tables", P), ("h_lens", P), ("h_out", P),
        ("d_query", P), ("d_key", P), ("d_value", P), ("d_slots", P), ("d_pairs", P), ("d_tables", P),
        ("d_lens", P), ("d_out", P), ("k_cache", P), ("v_cache", P), ("workspace", P), ("workspace_bytes", SZ),
        ("S", I), ("H", I), ("Hk", I), ("d", I), ("B", I), ("n_blocks", I), ("max_blocks_per_seq", I),
        ("max_context_len", I), ("max_pairs", I), ("partition_size", I),
        ("scale", F), ("kv_dtype", I), ("out_dtype", I),
    ]


# name -> (restype, argtypes); mirrors include/pa.h
SIGNATURES = {
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_version": (ctypes.c_char_p, []),
    "pa_decode_workspace_size": (SZ, [I, I, I, I, I, I]),
    "pa_decode": (I, [P, I, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, I, P, SZ, P]),
    "pa_decode_step": (I, [P, I, P, P, P, P, P, P, P, P, I, P, P, I, I, I, I, I, I, I, I, I, F, I, I, P, SZ, P]),
    "pa_decode_noalloc": (I, [P, I, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, I, P]),
    "pa_decode_default_partition": (I, [I, I, I]),
    "pa_prefill_workspace_size": (SZ, [I, I, I, I, I, I]),
    "pa_prefill": (I, [P, I, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, I, P, SZ, P]),
    "pa_workspace_error": (I, [P, IP, P]),
    "pa_selftest_wait_timeout": (I, [ctypes.c_uint, P, P]),
    "pa_combine": (I, [P, I, P, P, P, P, I, I, I, I, I, P]),
    "pa_cache_write": (I, [P, P, P, P, P, I, I, I, I, I, I, P]),
    "pa_copy_blocks": (I, [P, P, P, I, I, I, I, I, I, P]),
    "pa_swap_blocks": (I, [P, P, I, P, P, I, P, I, I, I, I, I, P]),
    "pa_step_create": (P, [ctypes.POINTER(StepDesc)]),
    "pa_step_run": (I, [P, P]),
    "pa_step_launch": (I, [P, P]),
    "pa_step_launch_async": (I, [P, P]),
    "pa_step_wait": (I, [P]),
    "pa_step_destroy": (None, [P]),
    "pa_alloc_create": (P, [I, I]),
    "pa_alloc_destroy": (None, [P]),
    "pa_alloc_block": (I, [P, I32P]),
    "pa_block_incref": (I, [P, ctypes.c_int32]),
    "pa_block_decref": (I, [P, ctypes.c_int32]),
    "pa_block_refcount": (I, [P, ctypes.c_int32]),
    "pa_alloc_num_free": (I, [P]),
    "pa_seq_create": (I, [P, I32P]),
    "pa_seq_fork": (I, [P, ctypes.c_int32, I32P]),
    "pa_seq_free": (I, [P, ctypes.c_int32]),
    # batch calls take their arrays as plain addresses (a tensor's data_ptr()): no per-call casts
    "pa_seq_fork_batch": (I, [P, P, I, P]),
    "pa_seq_free_batch": (I, [P, P, I]),
    "pa_seq_len": (I, [P, ctypes.c_int32]),
    "pa_seq_num_blocks": (I, [P, ctypes.c_int32]),
    "pa_seq_reserve_slots": (I, [P, ctypes.c_int32, I, I64P, I32P, IP]),
    "pa_seq_reserve_slots_batch": (I, [P, P, I, I, P, P, IP, IP]),
    "pa_build_block_tables": (I, [P, P, I, P, I, P]),
}

_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libpa.so not found at {LIB_PATH}; build it with `python -m paged_kv_cache_329_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
