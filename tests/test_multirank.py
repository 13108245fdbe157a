"""The N > 1 path of bench.py on CPU with gloo ranks: max-over-ranks timing, whole-job aggregation,
and the reference arm printing one line from rank 0 under torchrun."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench

    mine = [10.0 + rank, 5.0 - rank, 7.0 * (rank + 1)]
    got = bench.reduce_max(mine, world)
    q.put((rank, got, bench.aggregate_value(1e9, 10, world, got[0])))
    dist.destroy_process_group()


def test_reduce_max_and_aggregate_with_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, val in res:
        assert got == [11.0, 5.0, 14.0]                  # every rank sees the slowest rank's times
        assert abs(val - 2 * 1e9 * 10 / 11e-3 / 1e9) < 1e-6


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def _dying_worker(rank, world, port, q):
    import datetime
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    sys.path.insert(0, ROOT)
    import bench

    if rank == 1:
        raise SystemExit(3)                        # leaves between steps, before the timing collective
    t0 = time.time()
    try:
        bench.reduce_max([1.0], world)
        q.put(("returned", time.time() - t0))
    except Exception as e:                         # the survivor learns of it from the collective
        q.put(("error", time.time() - t0, type(e).__name__))


def test_rank_that_leaves_ends_the_collective_with_an_error():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dying_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert res[0] == "error", res                 # no hang, no silent result
    assert res[1] < 60.0
    assert procs[1].exitcode == 3
