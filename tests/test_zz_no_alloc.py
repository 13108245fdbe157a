"""pa_decode_noalloc: paged decode for callers that cannot allocate device memory.

Some callers (plugins whose host process owns the whole device-memory budget, serving loops that
must not allocate on the decode path) cannot hand the library a workspace.  This entry point
keeps its scratch in a device array inside libpa.  The GPU test calls it through the C ABI twice
in a row, on different inputs, and checks each result against pa_decode with a caller-provided
workspace, within the parity tolerance.  This file is collected last so that a failure here
comes after every other test has run.
"""
import ctypes
import math

import pytest
import torch

from paged_kv_cache_329_b200 import _native, api
from paged_kv_cache_329_b200 import workloads as W

TOL = {torch.float32: 1e-5, torch.float16: 2e-3, torch.bfloat16: 2e-3}
SCRATCH_BYTES = 32 << 20


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_329_b200 import build

    build.build()
    return _native.load()


def _noalloc(lib, case, out, max_c, P=0):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.pa_decode_noalloc(
        p(out), api.DTYPE[out.dtype], p(case.q), p(case.k_cache), p(case.v_cache), p(case.block_tables),
        p(case.context_lens), case.S, case.H, case.Hk, case.d, case.B, case.n_blocks,
        case.block_tables.shape[1], max_c, case.scale, api.DTYPE[case.q.dtype], P,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_rejects_sizes_beyond_the_scratch(lib):
    # 256 sequences of up to 8192 tokens at 32 heads need far more than 32 MiB of partials.
    S, H, Hk, d, max_c = 256, 32, 8, 128, 8192
    assert api.decode_workspace_size(S, H, Hk, d, max_c, 64) > SCRATCH_BYTES
    st = lib.pa_decode_noalloc(1 << 12, 0, 1 << 12, 1 << 12, 1 << 12, 1 << 12, 1 << 12, S, H, Hk, d, 16, 1000,
                               512, max_c, 0.1, 2, 64, None)
    assert st == api.PA_ERR_INVALID_ARG
    assert b"32 MiB" in lib.pa_last_error() or b"33554432" in lib.pa_last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_twice(lib):
    assert torch.cuda.is_available()
    cases = [
        W.paged_case("na1", W.lens_uniform(W.generator(31), 32, 1, 3000), 32, 8, 128, 16, torch.bfloat16, 31),
        W.paged_case("na2", W.lens_uniform(W.generator(32), 16, 1, 1500), 16, 16, 64, 8, torch.float16, 32),
    ]
    for case in cases:
        case = case.to("cuda")
        max_c = int(case.context_lens.max())
        assert api.decode_workspace_size(case.S, case.H, case.Hk, case.d, max_c, 0) <= SCRATCH_BYTES
        ref = api.pa_decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                            max_context_len=max_c, scale=case.scale, out_dtype=torch.float32)
        out = torch.full((case.S, case.H, case.d), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(lib, case, out, max_c) == api.PA_OK, lib.pa_last_error()
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        err = (out - ref).abs().max().item()
        assert err <= TOL[case.q.dtype], f"{case.name}: max-abs difference {err}"
