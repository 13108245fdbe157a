"""The C ABI loads without a GPU, exports every function include/pa.h declares, and rejects bad
arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_329_b200 import _native, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_329_b200 import build

    build.build()
    return _native.load()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_functions_are_exported(lib):
    names = _declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), f"{n} declared in pa.h but not exported"
        assert n in _native.SIGNATURES, f"{n} has no ctypes signature"


def test_version_and_error_strings(lib):
    assert "sm_100a" in api.version()
    assert isinstance(lib.pa_last_error(), bytes)


def _decode_status(lib, **kw):
    args = dict(out=1 << 12, out_dtype=0, q=1 << 12, k=1 << 12, v=1 << 12, bt=1 << 12, cl=1 << 12, S=2, H=8, Hk=2,
                d=128, B=16, n_blocks=10, mb=4, maxc=64, scale=0.1, kv=2, P=0, ws=1 << 12, wsb=1 << 30)
    args.update(kw)
    a = args
    return lib.pa_decode(a["out"], a["out_dtype"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["S"], a["H"], a["Hk"],
                         a["d"], a["B"], a["n_blocks"], a["mb"], a["maxc"], a["scale"], a["kv"], a["P"], a["ws"],
                         a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(H=6, Hk=4), api.PA_ERR_INVALID_ARG),        # H not a multiple of Hk
    (dict(H=6, Hk=2), api.PA_ERR_UNSUPPORTED),        # g = 3
    (dict(d=96), api.PA_ERR_UNSUPPORTED),
    (dict(B=12), api.PA_ERR_UNSUPPORTED),
    (dict(kv=7), api.PA_ERR_INVALID_ARG),
    (dict(P=100), api.PA_ERR_INVALID_ARG),            # not a multiple of 64
    (dict(mb=2), api.PA_ERR_INVALID_ARG),             # table too short for max_context_len
    (dict(q=(1 << 12) + 8), api.PA_ERR_INVALID_ARG),  # misaligned
    (dict(ws=(1 << 12) + 16), api.PA_ERR_INVALID_ARG),  # workspace not 256-aligned
    (dict(wsb=16), api.PA_ERR_INVALID_ARG),           # workspace too small
    (dict(out=0), api.PA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), api.PA_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments_on_host(lib, kw, status):
    assert _decode_status(lib, **kw) == status
    assert lib.pa_last_error()


def test_workspace_size_grows_with_context(lib):
    a = api.decode_workspace_size(4, 32, 8, 128, 1000, 512)
    b = api.decode_workspace_size(4, 32, 8, 128, 5000, 512)
    assert 0 < a < b
    assert api.default_partition(256, 8, 8192) % 64 == 0


def test_cache_ops_reject_bad_arguments(lib):
    assert lib.pa_cache_write(1 << 12, 1 << 12, 1 << 12, 1 << 12, 1 << 12, 4, 2, 100, 16, 8, 2, None) == api.PA_ERR_UNSUPPORTED
    assert lib.pa_cache_write(1 << 12, 1 << 12, 1 << 12, 1 << 12, 1 << 12, -1, 2, 128, 16, 8, 2, None) == api.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(1 << 12, (1 << 12) + 4, 1 << 12, 1, 2, 128, 16, 8, 2, None) == api.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(1 << 12, 1 << 12, 1 << 12, 0, 2, 128, 16, 8, 2, None) == api.PA_OK  # nothing to do
    assert lib.pa_combine(1 << 12, 0, 1 << 12, 1 << 12, 1 << 12, 1 << 12, 2, 4, 80, 3, 64, None) == api.PA_ERR_UNSUPPORTED


def test_default_partition_picks():
    # the largest of 8192 .. 256 with six units per SM (148 SMs without a device) at the length
    # bound, no larger than the power of two that holds the longest context; else 128
    from paged_kv_cache_329_b200 import api
    assert api.default_partition(256, 8, 8300) == 8192     # gqa8k: 2048 (seq, kv head) pairs
    assert api.default_partition(16, 8, 33000) == 4096     # long context: 8192 would leave 640 units
    assert api.default_partition(64, 40, 2200) == 4096     # 13B MHA: contexts <= 2200, no split
    assert api.default_partition(128, 8, 1400) == 2048     # shared prefix
    assert api.default_partition(256, 8, 100) == 256       # short contexts: one partition each
    assert api.default_partition(4, 8, 300) == 128         # few pairs: split for parallelism
    assert api.default_partition(1, 1, 5000) == 128
