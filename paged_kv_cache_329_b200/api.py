"""Python binding of libpa: argument marshalling only; every step runs in the C/CUDA library.

torch supplies device memory and the current CUDA stream.  Each function here checks tensor
placement and types, then calls the C entry point of the same name (include/pa.h) and raises
``PAError`` on a non-OK status.
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _native

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_NO_FREE_BLOCK, PA_ERR_CUDA, PA_ERR_UNSUPPORTED = range(5)
DTYPE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}


class PAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"[pa status {status}] {msg}")
        self.status = status


class NoFreeBlock(PAError):
    pass


def _check(status: int):
    if status != PA_OK:
        msg = _native.load().pa_last_error().decode(errors="replace")
        raise (NoFreeBlock if status == PA_ERR_NO_FREE_BLOCK else PAError)(status, msg)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _host_i32(x):
    """An input id array as a contiguous int32 CPU tensor (converted only when it is not one)."""
    if isinstance(x, torch.Tensor):
        if x.device.type == "cpu" and x.dtype == torch.int32 and x.is_contiguous():
            return x
        return x.to(device="cpu", dtype=torch.int32).contiguous()
    return torch.tensor(list(x), dtype=torch.int32)


def _check_host(t, dtype, n, what):
    """An output array the native code writes through a plain address: CPU, contiguous, dtype, size."""
    if t.device.type != "cpu" or t.dtype != dtype or not t.is_contiguous() or t.numel() < n:
        raise ValueError(f"{what} must be a contiguous {dtype} CPU tensor of at least {n} elements")


def _cuda(*ts):
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("expected contiguous CUDA tensors")


def version() -> str:
    return _native.load().pa_version().decode()


# ---- decode -------------------------------------------------------------------------------------

def default_partition(S: int, Hk: int, max_context_len: int) -> int:
    return _native.load().pa_decode_default_partition(S, Hk, max_context_len)


def decode_workspace_size(S, H, Hk, d, max_context_len, partition_size=0) -> int:
    return _native.load().pa_decode_workspace_size(S, H, Hk, d, max_context_len, partition_size)


def alloc_workspace(S, H, Hk, d, max_context_len, partition_size=0, device="cuda") -> torch.Tensor:
    n = decode_workspace_size(S, H, Hk, d, max_context_len, partition_size)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def pa_decode(q, k_cache, v_cache, block_tables, context_lens, *, max_context_len, scale=None, out=None,
              out_dtype=None, partition_size=0, workspace=None, stream=None):
    """Paged decode attention; returns out [S, H, d].  See pa_decode in include/pa.h."""
    _cuda(q, k_cache, v_cache, block_tables, context_lens)
    S, H, d = q.shape
    n_blocks, Hk, B, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape or q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise ValueError("shape/dtype mismatch between q and the caches")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if out is None:
        out = torch.empty((S, H, d), dtype=out_dtype or q.dtype, device=q.device)
    _cuda(out)
    if workspace is None:
        workspace = alloc_workspace(S, H, Hk, d, max_context_len, partition_size, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check(_native.load().pa_decode(
        _ptr(out), DTYPE[out.dtype], _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), S, H, Hk, d, B, n_blocks, block_tables.shape[1], int(max_context_len),
        float(scale), DTYPE[q.dtype], int(partition_size), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return out


def pa_decode_step(q, k_cache, v_cache, block_tables, context_lens, key, value, slot_mapping, pairs, *,
                   max_context_len, n_pairs=None, scale=None, out=None, out_dtype=None, partition_size=0,
                   workspace=None, stream=None):
    """One decode step: copy-on-write copies, slot writes, then decode, in fewer launches; returns out.
    pairs: int32 [max_pairs, 2] on the device; n_pairs: an int32 device tensor holding the count
    used (or None: every row of pairs).  See pa_decode_step in include/pa.h."""
    _cuda(q, k_cache, v_cache, block_tables, context_lens, key, value, slot_mapping, pairs)
    S, H, d = q.shape
    n_blocks, Hk, B, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape or q.dtype != k_cache.dtype or key.dtype != k_cache.dtype \
            or value.dtype != k_cache.dtype:
        raise ValueError("shape/dtype mismatch between q, key, value and the caches")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32 or pairs.dtype != torch.int32 \
            or slot_mapping.dtype != torch.int64:
        raise ValueError("block_tables, context_lens and pairs must be int32, slot_mapping int64")
    if n_pairs is not None:
        _cuda(n_pairs)
        if n_pairs.dtype != torch.int32:
            raise ValueError("n_pairs must be an int32 device tensor")
    if out is None:
        out = torch.empty((S, H, d), dtype=out_dtype or q.dtype, device=q.device)
    _cuda(out)
    if workspace is None:
        workspace = alloc_workspace(S, H, Hk, d, max_context_len, partition_size, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check(_native.load().pa_decode_step(
        _ptr(out), DTYPE[out.dtype], _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        _ptr(key), _ptr(value), _ptr(slot_mapping), key.shape[0], _ptr(pairs), _ptr(n_pairs), pairs.numel() // 2,
        S, H, Hk, d, B, n_blocks, block_tables.shape[1], int(max_context_len), float(scale), DTYPE[q.dtype],
        int(partition_size), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def prefill_workspace_size(S, H, Hk, d, max_context_len, max_q_len) -> int:
    return _native.load().pa_prefill_workspace_size(S, H, Hk, d, int(max_context_len), int(max_q_len))


def pa_prefill(q, q_start, k_cache, v_cache, block_tables, context_lens, *, max_context_len, max_q_len,
               scale=None, out=None, out_dtype=None, workspace=None, stream=None):
    """Causal paged attention for several query tokens per sequence (prefill chunks and decode tokens
    in one batch); returns out [T, H, d].  See pa_prefill in include/pa.h."""
    _cuda(q, q_start, k_cache, v_cache, block_tables, context_lens)
    T, H, d = q.shape
    n_blocks, Hk, B, d2 = k_cache.shape
    S = context_lens.numel()
    if d2 != d or q.dtype != k_cache.dtype or q_start.dtype != torch.int32 or q_start.numel() != S + 1:
        raise ValueError("shape/dtype mismatch")
    if out is None:
        out = torch.empty((T, H, d), dtype=out_dtype or q.dtype, device=q.device)
    if workspace is None:
        n = prefill_workspace_size(S, H, Hk, d, max_context_len, max_q_len)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check(_native.load().pa_prefill(
        _ptr(out), DTYPE[out.dtype], _ptr(q), _ptr(q_start), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), S, H, Hk, d, B, n_blocks, block_tables.shape[1], int(max_context_len), int(max_q_len),
        float(scale), DTYPE[q.dtype], _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def workspace_error(workspace, stream=None) -> int:
    flags = ctypes.c_int(0)
    _check(_native.load().pa_workspace_error(_ptr(workspace), ctypes.byref(flags), _stream(stream)))
    return flags.value


def pa_combine(part_o, part_m, part_l, context_lens, partition_size, *, out=None, out_dtype=torch.float32,
               stream=None):
    """Log-sum-exp merge of per-partition states; see pa_combine in include/pa.h."""
    _cuda(part_o, part_m, part_l, context_lens)
    S, H, max_parts, d = part_o.shape
    if out is None:
        out = torch.empty((S, H, d), dtype=out_dtype, device=part_o.device)
    _check(_native.load().pa_combine(
        _ptr(out), DTYPE[out.dtype], _ptr(part_o), _ptr(part_m), _ptr(part_l), _ptr(context_lens),
        S, H, d, max_parts, int(partition_size), _stream(stream)))
    return out


# ---- cache maintenance --------------------------------------------------------------------------

def pa_cache_write(k_cache, v_cache, key, value, slot_mapping, stream=None):
    _cuda(k_cache, v_cache, key, value, slot_mapping)
    n_blocks, Hk, B, d = k_cache.shape
    if slot_mapping.dtype != torch.int64 or key.dtype != k_cache.dtype or value.dtype != k_cache.dtype:
        raise ValueError("slot_mapping must be int64 and key/value must match the cache type")
    _check(_native.load().pa_cache_write(
        _ptr(k_cache), _ptr(v_cache), _ptr(key), _ptr(value), _ptr(slot_mapping), key.shape[0], Hk, d, B,
        n_blocks, DTYPE[k_cache.dtype], _stream(stream)))


def pa_copy_blocks(k_cache, v_cache, pairs, stream=None):
    _cuda(k_cache, v_cache, pairs)
    n_blocks, Hk, B, d = k_cache.shape
    if pairs.dtype != torch.int32:
        raise ValueError("pairs must be int32 [P, 2]")
    _check(_native.load().pa_copy_blocks(
        _ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.numel() // 2, Hk, d, B, n_blocks,
        DTYPE[k_cache.dtype], _stream(stream)))


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, pairs, stream=None):
    """Whole-block copies between the device cache and a pinned host pool (either direction)."""
    for t in (dst_k, dst_v, src_k, src_v, pairs):
        if not t.is_contiguous() or not (t.is_cuda or t.is_pinned()):
            raise ValueError("pools and pairs must be contiguous CUDA or pinned host tensors")
    n_dst, Hk, B, d = dst_k.shape
    if src_k.shape[1:] != dst_k.shape[1:] or src_k.dtype != dst_k.dtype or pairs.dtype != torch.int32:
        raise ValueError("pools must share the block layout and type; pairs int32 [P, 2]")
    _check(_native.load().pa_swap_blocks(
        _ptr(dst_k), _ptr(dst_v), n_dst, _ptr(src_k), _ptr(src_v), src_k.shape[0], _ptr(pairs),
        pairs.numel() // 2, Hk, d, B, DTYPE[dst_k.dtype], _stream(stream)))


# ---- a decode step as one CUDA graph -------------------------------------------------------------

class DecodeStep:
    """pa_step_*: the step's H2D copies, COW copy, cache write, decode and D2H of o, captured once.

    Fill the pinned host tensors (h_query, h_key, h_value, h_slots, h_pairs, h_n_pairs, h_tables,
    h_lens) before each run(); the output is in h_out afterwards.
    """

    def __init__(self, k_cache, v_cache, S, H, max_blocks_per_seq, max_context_len, *, max_pairs=None,
                 out_dtype=None, scale=None, partition_size=0):
        _cuda(k_cache, v_cache)
        n_blocks, Hk, B, d = k_cache.shape
        dt, dev = k_cache.dtype, k_cache.device
        out_dtype = out_dtype or dt
        max_pairs = S if max_pairs is None else max_pairs
        # Every input lives at the same offset in one pinned block and one device block, so the
        # captured step moves them with a single host->device transfer.
        mp = max(max_pairs, 1)
        fields = [("query", (S, H, d), dt), ("key", (S, Hk, d), dt), ("value", (S, Hk, d), dt),
                  ("slots", (S,), torch.int64), ("pairs", (2 * mp + 4,), torch.int32),
                  ("tables", (S, max_blocks_per_seq), torch.int32), ("lens", (S,), torch.int32)]
        offs, total = {}, 0
        for name, shape, t in fields:
            offs[name] = total
            total += -(-math.prod(shape) * torch.empty((), dtype=t).element_size() // 256) * 256
        self._h_block = torch.zeros(total, dtype=torch.uint8).pin_memory()
        self._d_block = torch.zeros(total, dtype=torch.uint8, device=dev)
        for name, shape, t in fields:
            n = math.prod(shape) * torch.empty((), dtype=t).element_size()
            setattr(self, "h_" + name, self._h_block[offs[name]: offs[name] + n].view(t).view(shape))
            setattr(self, "d_" + name, self._d_block[offs[name]: offs[name] + n].view(t).view(shape))
        self.h_n_pairs = self.h_pairs[2 * mp: 2 * mp + 1]           # the count sits right after the pairs
        self.h_pairs = self.h_pairs[: 2 * mp].view(mp, 2)
        self.h_out = torch.empty((S, H, d), dtype=out_dtype).pin_memory()
        self.d_out = torch.zeros((S, H, d), dtype=out_dtype, device=dev)
        self.h_slots.fill_(-1)
        self.workspace = alloc_workspace(S, H, Hk, d, max_context_len, partition_size, dev)
        self.k_cache, self.v_cache = k_cache, v_cache
        vp = lambda t: t.data_ptr()
        desc = _native.StepDesc(
            vp(self.h_query), vp(self.h_key), vp(self.h_value), vp(self.h_slots), vp(self.h_pairs),
            vp(self.h_n_pairs), vp(self.h_tables), vp(self.h_lens), vp(self.h_out),
            vp(self.d_query), vp(self.d_key), vp(self.d_value), vp(self.d_slots), vp(self.d_pairs),
            vp(self.d_tables), vp(self.d_lens), vp(self.d_out), vp(k_cache), vp(v_cache), vp(self.workspace),
            self.workspace.numel(), S, H, Hk, d, B, n_blocks, max_blocks_per_seq, max_context_len, max_pairs,
            partition_size, float(1.0 / math.sqrt(d) if scale is None else scale), DTYPE[dt], DTYPE[out_dtype])
        self._lib = _native.load()
        self._h = self._lib.pa_step_create(ctypes.byref(desc))
        if not self._h:
            raise PAError(PA_ERR_INVALID_ARG, self._lib.pa_last_error().decode())
        self.h2d_bytes = self._h_block.numel()
        self.d2h_bytes = self.h_out.numel() * self.h_out.element_size()

    def set_pairs(self, pairs):
        n = int(pairs.shape[0]) if pairs is not None else 0
        if n > self.h_pairs.shape[0]:
            raise ValueError("more copy-on-write pairs than max_pairs")
        if n:
            self.h_pairs[:n].copy_(pairs)
        self.h_n_pairs[0] = n

    def run(self, stream=None):
        _check(self._lib.pa_step_run(self._h, _stream(stream)))
        return self.h_out

    def launch(self, stream=None):
        """Enqueue the step and return; h_out is valid once the stream reaches it."""
        _check(self._lib.pa_step_launch(self._h, _stream(stream)))

    def launch_async(self, stream=None):
        """Enqueue the step with its input and output copies on the step's own copy streams, so
        that they overlap neighbouring steps' kernels.  Refill the host inputs and read h_out only
        after wait()."""
        _check(self._lib.pa_step_launch_async(self._h, _stream(stream)))

    def wait(self):
        """Block until the output of the last launch_async() is in h_out."""
        _check(self._lib.pa_step_wait(self._h))
        return self.h_out

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._lib.pa_step_destroy(h)
            self._h = None


# ---- host block manager -------------------------------------------------------------------------

class BlockManager:
    """Reference-counted block pool with sequences (pa_alloc_* / pa_seq_* in include/pa.h)."""

    def __init__(self, n_blocks: int, block_size: int):
        self._lib = _native.load()
        self._h = self._lib.pa_alloc_create(n_blocks, block_size)
        if not self._h:
            raise PAError(PA_ERR_INVALID_ARG, self._lib.pa_last_error().decode())
        self.n_blocks = n_blocks
        self.B = block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._lib.pa_alloc_destroy(h)
            self._h = None

    def alloc_block(self) -> int:
        b = ctypes.c_int32()
        _check(self._lib.pa_alloc_block(self._h, ctypes.byref(b)))
        return b.value

    def incref(self, b: int):
        _check(self._lib.pa_block_incref(self._h, b))

    def decref(self, b: int):
        _check(self._lib.pa_block_decref(self._h, b))

    def refcount(self, b: int) -> int:
        return self._lib.pa_block_refcount(self._h, b)

    def num_free(self) -> int:
        return self._lib.pa_alloc_num_free(self._h)

    def seq_create(self) -> int:
        s = ctypes.c_int32()
        _check(self._lib.pa_seq_create(self._h, ctypes.byref(s)))
        return s.value

    def seq_fork(self, parent: int) -> int:
        s = ctypes.c_int32()
        _check(self._lib.pa_seq_fork(self._h, parent, ctypes.byref(s)))
        return s.value

    def seq_free(self, sid: int):
        _check(self._lib.pa_seq_free(self._h, sid))

    def seq_fork_batch(self, parents):
        """Fork each parent in order; returns the children as an int32 tensor."""
        p = _host_i32(parents)
        kids = torch.empty(p.numel(), dtype=torch.int32)
        _check(self._lib.pa_seq_fork_batch(self._h, p.data_ptr(), p.numel(), kids.data_ptr()))
        return kids

    def seq_free_batch(self, seq_ids):
        ids = _host_i32(seq_ids)
        _check(self._lib.pa_seq_free_batch(self._h, ids.data_ptr(), ids.numel()))

    def seq_len(self, sid: int) -> int:
        return self._lib.pa_seq_len(self._h, sid)

    def seq_num_blocks(self, sid: int) -> int:
        return self._lib.pa_seq_num_blocks(self._h, sid)

    def reserve_slots(self, sid: int, n_new: int):
        """Returns (slots: list[int], cow_pairs: list[(src, dst)])."""
        slots = (ctypes.c_int64 * max(n_new, 1))()
        pairs = (ctypes.c_int32 * 2)()
        n_cow = ctypes.c_int(0)
        _check(self._lib.pa_seq_reserve_slots(self._h, sid, n_new, slots, pairs, ctypes.byref(n_cow)))
        return list(slots[:n_new]), [(pairs[2 * i], pairs[2 * i + 1]) for i in range(n_cow.value)]

    def reserve_slots_batch(self, seq_ids, n_new: int = 1, slots=None, pairs=None):
        """One step for a batch: n_new slots per sequence.  Returns (slots int64 [S*n_new] tensor,
        pairs int32 [n_cow, 2] tensor).  `slots`/`pairs` may be preallocated (pinned) CPU tensors."""
        ids = _host_i32(seq_ids)
        S = ids.numel()
        if slots is None:
            slots = torch.empty(S * n_new, dtype=torch.int64)
        if pairs is None:
            pairs = torch.empty((max(S, 1), 2), dtype=torch.int32)
        _check_host(slots, torch.int64, S * n_new, "slots")
        _check_host(pairs, torch.int32, 2 * max(S, 1), "pairs")
        n_cow, n_done = ctypes.c_int(0), ctypes.c_int(0)
        _check(self._lib.pa_seq_reserve_slots_batch(self._h, ids.data_ptr(), S, n_new, slots.data_ptr(),
                                                    pairs.data_ptr(), ctypes.byref(n_cow), ctypes.byref(n_done)))
        return slots, pairs[: n_cow.value]

    def build_block_tables(self, seq_ids, max_blocks_per_seq: int, tables=None, lens=None):
        """Returns (tables int32 [S, max_blocks] CPU tensor, context_lens int32 [S] CPU tensor)."""
        ids = _host_i32(seq_ids)
        S = ids.numel()
        if tables is None:
            tables = torch.empty((S, max_blocks_per_seq), dtype=torch.int32)
        if lens is None:
            lens = torch.empty((S,), dtype=torch.int32)
        _check_host(tables, torch.int32, S * max_blocks_per_seq, "tables")
        _check_host(lens, torch.int32, S, "lens")
        _check(self._lib.pa_build_block_tables(self._h, ids.data_ptr(), S, tables.data_ptr(), max_blocks_per_seq,
                                               lens.data_ptr()))
        return tables, lens
