"""Paged decode attention for B200 (sm_100a): Python binding of the C ABI in include/pa.h.

    from paged_kv_cache_329_b200 import pa_decode, pa_cache_write, pa_copy_blocks, BlockManager

The entry points load the in-tree libpa.so on first use and raise if it is missing; nothing here
computes on the CPU.
"""
from .api import (  # noqa: F401
    BlockManager,
    DecodeStep,
    NoFreeBlock,
    PAError,
    alloc_workspace,
    decode_workspace_size,
    default_partition,
    pa_cache_write,
    pa_combine,
    pa_copy_blocks,
    pa_decode,
    pa_decode_step,
    pa_prefill,
    pa_swap_blocks,
    version,
    workspace_error,
)
