"""The measurement arithmetic of bench.py, checked by hand on tiny cases (CPU only)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _Shape:
    """Only the attributes the byte formulas read."""
    S, H, Hk, d, B, es, P = 2, 4, 2, 8, 4, 2, 8


def test_step_bytes_by_hand():
    # lens 5 and 9: K and V of 14 tokens x 2 kv heads x 8 dims x 2 bytes, twice
    wl = _Shape()
    decode, step, kv = bench.Workload.step_bytes(wl, [5, 9], n_pairs=1)
    assert kv == 14 * 2 * 8 * 2 * 2
    q_o = 2 * 4 * 8 * 2 * 2                       # q read and o written, 2 seqs x 4 heads x 8 dims
    table = 4 * (2 + 3)                          # ceil(5/4) + ceil(9/4) block ids
    assert decode == kv + q_o + table + 4 * 2    # + the two lengths
    write = 2 * (2 * 2 * 8 * 2 * 2) + 8 * 2      # new K and V read and written, + slot ids
    copy = 1 * 2 * (2 * 4 * 8 * 2) * 2           # one pair: K and V blocks read and written
    assert step == decode + write + copy


def test_touched_bytes_by_hand():
    # whole blocks (8 and 12 slots) and the partials of the one split sequence (9 > P = 8: 2 parts)
    wl = _Shape()
    got = bench.Workload.touched_bytes(wl, [5, 9])
    blocks = 2 + 3
    kv = blocks * 4 * 2 * 8 * 2 * 2
    partials = 2 * 2 * 4 * (8 + 2) * 4           # written then read: 2 parts x 4 heads x (o, m, l)
    assert got == kv + 2 * 4 * 8 * 2 * 2 + 4 * blocks + 4 * 2 + partials


def test_aggregate_value_and_reduce_max_single_rank():
    assert abs(bench.aggregate_value(1e9, 10, 1, 2.0) - 1e9 * 10 / 2e-3 / 1e9) < 1e-9
    assert bench.reduce_max([3.0, 1.0], 1) == [3.0, 1.0]


def test_clock_sampler_windows():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.proc, c.windows = None, []
    c.samples = [(10.0, 1900.0, 1965.0, []), (10.05, 1950.0, 1965.0, ["sw_power_cap"]),
                 (10.10, 1960.0, 1965.0, []), (11.0, 1000.0, 1965.0, ["hw_slowdown"])]
    # a window holding two samples takes exactly those
    c.windows = [(10.04, 10.11)]
    c.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0})()
    c.thread = type("T", (), {"join": lambda self, timeout=None: None})()
    out = c.finish()
    assert out["samples"] == 2 and out["sm_mhz"] == 1955.0 and out["reasons"] == ["sw_power_cap"]
    # a window shorter than the sampling interval takes the samples nearest to it
    c.windows = [(10.06, 10.07)]
    out = c.finish()
    assert out["samples"] == 2 and out["reasons"] == ["sw_power_cap"] and "hw_slowdown" not in out["reasons"]


def test_profiled_traffic_matches_the_committed_sources():
    # the roofline's traffic comes from the committed ncu summaries only while their recorded code
    # hashes are those of the current sources; a kernel edit without a new capture drops it to null
    class A:
        partition = block_size = seqs = 0
    for wl in bench.PROFILED:
        A.workload = wl
        t = bench.profiled_traffic(A)
        assert t is not None and t > 1e8, f"{wl}: the profile's code hashes do not match the sources"
    A.workload, A.seqs = "gqa8k_bf16", 64
    assert bench.profiled_traffic(A) is None          # another workload than the one captured
    A.workload, A.seqs = "long_bf16", 0
    assert bench.profiled_traffic(A) is None


def test_code_hash_ignores_comments(tmp_path):
    a, b, c = tmp_path / "a.cu", tmp_path / "b.cu", tmp_path / "c.cu"
    a.write_text("int f() {\n  return 1;  // one\n}\n")
    b.write_text("/* header */\nint f() {\n\n  return 1;\n}\n")
    c.write_text("int f() {\n  return 2;\n}\n")
    assert bench.code_sha256(str(a)) == bench.code_sha256(str(b)) != bench.code_sha256(str(c))
