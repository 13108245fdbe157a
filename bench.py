"""Benchmark of the paged-decode hot path on B200; prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pa|reference] [--workload NAME]

A step is one pass of the whole path over one batch of the workload:
  host block manager (one slot per sequence, copy-on-write pairs, packed block tables)
  -> pa_copy_blocks (the step's COW pairs) -> pa_cache_write (one new token per sequence)
  -> pa_decode (plan, split-K decode, log-sum-exp combine).
`value` is the device-timed throughput of K such steps with every input already in HBM (the
host-side block management for the step is done before the timed region); `e2e` runs the same
steps through the Python API from pinned host buffers, with the block manager, the host->device
copies of the step's inputs and the device->host read of the outputs inside the timed region.

The metric is effective KV bandwidth: the bytes the step must move by definition (every valid
cached token's K and V once, q, o, block tables, lengths, the new tokens' K/V read and written,
the COW blocks read and written), divided by the step time.

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica of the workload
(sequence-sharded serving, no collective on the data path); value = all ranks' bytes / the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_329_b200 import api  # noqa: E402
from paged_kv_cache_329_b200 import workloads as W  # noqa: E402

METRIC = "paged decode-attn effective KV GB/s (% of B200 HBM peak); seqs/s per step"
L2_BYTES = 126e6   # B200 L2
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e nominal bandwidth (about 8 TB/s), beside the measured copy peak
E2E_DEPTH = 3      # decode steps in flight in the end-to-end leg


# ---- workload -----------------------------------------------------------------------------------

WORKLOADS = {
    "gqa8k_bf16": dict(S=256, H=32, Hk=8, d=128, B=16, dtype=torch.bfloat16, lens=lambda: W.gqa8k_lens(256),
                       desc="GQA bf16 decode at 8k: 256 seqs, 32 q / 8 kv heads, d=128, B=16, context lognormal "
                            "(median 1024, sigma 1.0) clipped to [16, 8192], shuffled block pool"),
    "mha13b_fp16": dict(S=64, H=40, Hk=40, d=128, B=16, dtype=torch.float16,
                        lens=lambda: W.lens_uniform(W.generator(2), 64, 1, 2048),
                        desc="13B-style MHA fp16: 64 seqs, 40 heads, d=128, B=16, context U[1,2048]"),
    "shared_prefix_bf16": dict(S=128, H=32, Hk=8, d=128, B=16, dtype=torch.bfloat16, lens=None,
                               desc="shared-prefix sampling and beam search, bf16: 32 requests x 4 sequences share "
                                    "a 1024-token prompt (64 blocks at ref count 4), tails U[0,256]; every step "
                                    "each sequence forks from a seeded parent among its request's 4, so shared "
                                    "partial tail blocks are copied on write"),
    "shared_prefix_partial_bf16": dict(S=128, H=32, Hk=8, d=128, B=16, dtype=torch.bfloat16, lens=None,
                                       desc="shared-prefix sampling with a partial last prompt block, bf16: 32 "
                                            "requests x 4 sequences share a 1031-token prompt (64 full blocks and "
                                            "one of 7 tokens, all at ref count 4) and start generating; the first "
                                            "step copies the partial block for 3 of each request's 4 sequences, "
                                            "then beam-style forks as in the shared-prefix workload"),
    "tiny_fp32": dict(S=4, H=8, Hk=8, d=64, B=16, dtype=torch.float32,
                      lens=lambda: W.lens_uniform(W.generator(1), 4, 1, 200),
                      desc="tiny fp32 paged decode: 4 seqs, 8 q heads = 8 kv heads, d=64, B=16, context U[1,200]"),
    "long_bf16": dict(S=16, H=64, Hk=8, d=128, B=16, dtype=torch.bfloat16,
                      lens=lambda: W.lens_uniform(W.generator(5), 16, 16384, 32768),
                      desc="long-context bf16: 16 seqs, 64 q / 8 kv heads, d=128, B=16, context U[16384,32768]"),
}


class Workload:
    """Sequences in a native block manager over a shuffled pool, random K/V in HBM."""

    def __init__(self, name, device, seed_offset=0, growth_steps=0, partition=0, block_size=0, seqs=0):
        cfg = dict(WORKLOADS[name])
        if block_size:
            cfg["B"] = block_size
            cfg["desc"] = cfg["desc"].replace("B=16", f"B={block_size}")
        if seqs:       # the first `seqs` sequences only (a smaller case of the same workload, for profiling)
            lens_fn = cfg["lens"]
            cfg["lens"] = (lambda: lens_fn()[:seqs]) if lens_fn else None
            cfg["S"] = seqs
            cfg["desc"] += f" (first {seqs} sequences only)"
        self.name, self.cfg = name, cfg
        self.S, self.H, self.Hk, self.d, self.B, self.dtype = (cfg[k] for k in ("S", "H", "Hk", "d", "B", "dtype"))
        self.es = torch.finfo(self.dtype).bits // 8
        lens = self._lengths()                 # context length of each sequence after this step's token
        B = self.B
        need = self._blocks_needed(lens)
        self.n_blocks = math.ceil(1.25 * need) + self.S * (growth_steps // B + 2)
        self.mgr = api.BlockManager(self.n_blocks, B)
        # Shuffle the free stack: take every block, release them in a seeded random order.
        g = torch.Generator().manual_seed(4242 + seed_offset)
        blocks = [self.mgr.alloc_block() for _ in range(self.n_blocks)]
        for i in torch.randperm(self.n_blocks, generator=g).tolist():
            self.mgr.decref(blocks[i])
        self.seqs = torch.empty(self.S, dtype=torch.int32)
        self._make_sequences(lens)
        self.max_blocks = max(lens) // B + growth_steps // B + 4
        self.max_c = max(lens) + growth_steps + 1
        gen = torch.Generator(device=device).manual_seed(77 + seed_offset)
        shape = (self.n_blocks, self.Hk, B, self.d)
        self.k_cache = torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(self.dtype)
        self.v_cache = torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(self.dtype)
        self.device = device
        self.P = partition or api.default_partition(self.S, self.Hk, self.max_c)
        self.workspace = api.alloc_workspace(self.S, self.H, self.Hk, self.d, self.max_c, self.P, device)

    def _lengths(self):
        return self.cfg["lens"]().tolist()

    def _blocks_needed(self, lens):
        return sum(-(-c // self.B) for c in lens)

    def _make_sequences(self, lens):
        for i, c in enumerate(lens):
            sid = self.mgr.seq_create()
            self.mgr.reserve_slots(sid, c - 1)  # tokens cached before this step
            self.seqs[i] = sid

    def trajectory(self, n_steps):
        """Host block management for n_steps consecutive steps, uploaded to HBM."""
        steps = []
        for _ in range(n_steps):
            slots, pairs, tables, lens = self.host_step()
            dev = self.device
            steps.append(dict(slots=slots.to(dev), pairs=pairs.to(dev), tables=tables.to(dev), lens=lens.to(dev),
                              n_pairs=pairs.shape[0], lens_host=lens.tolist()))
        return steps

    def host_step(self, slots=None, pairs=None, tables=None, lens=None):
        """One step of host block management: a slot per sequence, COW pairs, packed tables."""
        slots, pairs = self.mgr.reserve_slots_batch(self.seqs, 1, slots, pairs)
        tables, lens = self.mgr.build_block_tables(self.seqs, self.max_blocks, tables, lens)
        return slots, pairs, tables, lens

    def touched_bytes(self, lens):
        """Bytes a decode launch moves counting whole blocks (the last block's unused slots too) and
        the split-K partials (fp32 m, l and o written by the decode kernel, read by the combine)."""
        S, H, Hk, d, B, es, P = self.S, self.H, self.Hk, self.d, self.B, self.es, self.P
        lens = [int(c) for c in lens]
        blocks = sum(-(-c // B) for c in lens)
        parts = sum(-(-c // P) for c in lens if c > P)          # partitions of split sequences
        return (blocks * B * Hk * d * 2 * es + S * H * d * es * 2 + 4 * blocks + 4 * S
                + 2 * parts * H * (d + 2) * 4)

    def step_bytes(self, lens, n_pairs):
        S, H, Hk, d, B, es = self.S, self.H, self.Hk, self.d, self.B, self.es
        lens = [int(c) for c in lens]
        kv = sum(lens) * Hk * d * 2 * es
        decode = kv + S * H * d * es * 2 + 4 * sum(-(-c // B) for c in lens) + 4 * S
        write = 2 * (S * Hk * d * es * 2) + 8 * S
        copy = n_pairs * 2 * (Hk * B * d * es) * 2
        return decode, decode + write + copy, kv


class SharedPrefixWorkload(Workload):
    """32 requests x 4 beams over a shared 1024-token prompt; beam-style forks every step."""

    REQUESTS, WIDTH, PROMPT, TAIL_MAX = 32, 4, 1024, 256

    def __init__(self, name, device, seed_offset=0, growth_steps=0, partition=0, block_size=0, seqs=0):
        self.rnd = torch.Generator().manual_seed(4 + seed_offset)
        if seqs:
            raise ValueError("the shared-prefix workloads keep their 32 requests x 4 sequences")
        super().__init__(name, device, seed_offset, growth_steps + 64, partition, block_size)

    def _lengths(self):
        tails = torch.randint(0, self.TAIL_MAX + 1, (self.REQUESTS * self.WIDTH,), generator=self.rnd)
        self.tails = tails.tolist()
        return [self.PROMPT + t + 1 for t in self.tails]

    def _blocks_needed(self, lens):
        B = self.B
        prompt = self.REQUESTS * (self.PROMPT // B)
        tails = sum(-(-(c - self.PROMPT) // B) + 1 for c in lens)
        return prompt + 2 * tails

    def _make_sequences(self, lens):
        self.groups = []
        i = 0
        for r in range(self.REQUESTS):
            root = self.mgr.seq_create()
            self.mgr.reserve_slots(root, self.PROMPT)
            beams = [root] + [self.mgr.seq_fork(root) for _ in range(self.WIDTH - 1)]
            for b in beams:
                self.mgr.reserve_slots(b, lens[i] - 1 - self.PROMPT)
                self.seqs[i] = b
                i += 1
            self.groups.append(beams)

    def host_step(self, slots=None, pairs=None, tables=None, lens=None):
        # every beam picks a parent among its request's beams; children share the parent's blocks
        beams = self.seqs.view(self.REQUESTS, self.WIDTH)
        choice = torch.randint(0, self.WIDTH, (self.REQUESTS, self.WIDTH), generator=self.rnd)
        parents = torch.gather(beams, 1, choice).reshape(-1).to(torch.int32)
        kids = self.mgr.seq_fork_batch(parents)
        self.mgr.seq_free_batch(self.seqs)
        self.seqs.copy_(kids)
        return super().host_step(slots, pairs, tables, lens)

    def unique_kv_bytes(self, tables, lens):
        used = set()
        for s in range(self.S):
            nb = -(-int(lens[s]) // self.B)
            used.update(tables[s, :nb].tolist())
        return len(used) * self.Hk * self.B * self.d * 2 * self.es


class SharedPrefixPartialWorkload(SharedPrefixWorkload):
    """The shared-prefix workload with a 1031-token prompt (its last block holds 7 tokens and is
    shared by the request's 4 sequences) and no generated tokens yet: the first step's writes copy
    that block for 3 of the 4 sequences, and the last one writes into it in place."""

    PROMPT, TAIL_MAX = 1031, 0


def make_workload(name, device, seed_offset=0, growth_steps=0, partition=0, block_size=0, seqs=0):
    cls = {"shared_prefix_bf16": SharedPrefixWorkload,
           "shared_prefix_partial_bf16": SharedPrefixPartialWorkload}.get(name, Workload)
    return cls(name, device, seed_offset, growth_steps, partition, block_size, seqs)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def code_sha256(path):
    """sha256 of a C/C++/CUDA source with its comments and blank lines removed, so that a comment
    edit does not count as a change of the code a profile was taken on."""
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.split("\n")]
    return hashlib.sha256("\n".join(ln for ln in lines if ln.strip()).encode()).hexdigest()


PROFILED = {  # workload -> (ncu summary, sources its dominant kernel is built from)
    "gqa8k_bf16": ("decode_kernel_gqa8k_bf16.md", ("pa_decode.cu", "pa_device.cuh")),
    "prefill_mixed_bf16": ("prefill_umma_kernel_mixed_bf16.md", ("pa_prefill.cu", "pa_device.cuh")),
}


def profiled_traffic(args):
    """DRAM bytes per launch of the workload's dominant kernel from the committed ncu summary, if
    the code it was captured on is the current code (comments aside) and the run is the workload it
    was captured on (library-default partition and B, all sequences)."""
    if args.workload not in PROFILED or args.partition or args.block_size or args.seqs:
        return None
    name, files = PROFILED[args.workload]
    path = os.path.join(ROOT, "profiles", name)
    srcs = [os.path.join(ROOT, "paged_kv_cache_329_b200", "csrc", f) for f in files]
    try:
        text = open(path).read()
        want = dict(re.findall(r"code_sha256\((\S+)\):\s*([0-9a-f]{64})", text))
        t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text).group(1)
        ok = all(want.get(os.path.basename(f)) == code_sha256(f) for f in srcs)
        return float(t) if ok else None
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed loops run.  A reader
    thread collects the samples; the constructor returns once sampling has started, and a timed
    window shorter than the sampling interval takes the samples nearest to it."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index):
        import threading

        self.proc, self.windows, self.samples = None, [], []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 5.0 and self.proc.poll() is None:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                whole, _, frac = f[0].partition(".")
                ts = time.mktime(time.strptime(whole, "%Y/%m/%d %H:%M:%S")) + (float("0." + frac) if frac else 0.0)
                sm, mx = float(f[1]), float(f[2])
            except Exception:
                continue
            self.samples.append((ts, sm, mx, [n for n, v in zip(self.NAMES, f[4:8]) if v.lower() == "active"]))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def finish(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)
        picked = []
        for a, b in self.windows:
            inside = [x for x in self.samples if a <= x[0] <= b]
            if not inside and self.samples:     # window shorter than the sampling interval
                inside = sorted(self.samples, key=lambda x: min(abs(x[0] - a), abs(x[0] - b)))[:2]
            picked += inside
        if not picked:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({n for x in picked for n in x[3]})
        return {"sm_mhz": statistics.median(x[1] for x in picked), "sm_max_mhz": max(x[2] for x in picked),
                "reasons": reasons, "samples": len(picked)}


def reduce_max(values, world, device="cpu"):
    """Element-wise maximum over ranks (every rank gets it); the slowest rank sets the time."""
    t = torch.tensor(values, device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def aggregate_value(bytes_per_rank_step, steps, world, max_ms):
    """Whole-job GB/s: all ranks' bytes over the slowest rank's time."""
    return world * bytes_per_rank_step * steps / (max_ms * 1e-3) / 1e9


# ---- the GPU arm ----------------------------------------------------------------------------------

def run_pa(args, rank, world, local_rank):
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    K, Wm = args.steps, args.warmup
    e2e_steps = args.e2e_steps
    n_traj = 32 if args.workload.startswith("shared_prefix") else 1
    wl = make_workload(args.workload, dev, seed_offset=rank, growth_steps=e2e_steps + Wm + n_traj + 2,
                       partition=args.partition, block_size=args.block_size, seqs=args.seqs)
    S, H, Hk, d = wl.S, wl.H, wl.Hk, wl.d
    gen = torch.Generator(device=dev).manual_seed(99 + rank)
    q = torch.randn((S, H, d), generator=gen, device=dev).to(wl.dtype)
    key = torch.randn((S, Hk, d), generator=gen, device=dev).to(wl.dtype)
    val = torch.randn((S, Hk, d), generator=gen, device=dev).to(wl.dtype)
    out = torch.empty((S, H, d), dtype=wl.dtype, device=dev)

    # Host block management for a fixed trajectory of steps, done before timing; the timed loop
    # replays it with every input in HBM (one step for the decode-only workloads).
    traj = wl.trajectory(n_traj)
    for st in traj:
        st["decode_bytes"], st["step_bytes"], st["kv_bytes"] = wl.step_bytes(st["lens_host"], st["n_pairs"])
    max_parts = -(-wl.max_c // wl.P)
    launches = [2 + (1 if max_parts > 1 else 0) for st in traj]      # prologue, decode, combine

    def device_step(st):
        """The step as one call: copies, writes and the plan in one kernel, then decode (and combine)."""
        api.pa_decode_step(q, wl.k_cache, wl.v_cache, st["tables"], st["lens"], key, val, st["slots"], st["pairs"],
                           max_context_len=wl.max_c, out=out, partition_size=wl.P, workspace=wl.workspace)

    def separate_calls(st, evs):
        """The same step as three calls, timed call by call (the decode call gives the roofline)."""
        evs[0].record()
        if st["n_pairs"]:
            api.pa_copy_blocks(wl.k_cache, wl.v_cache, st["pairs"])
        evs[1].record()
        api.pa_cache_write(wl.k_cache, wl.v_cache, key, val, st["slots"])
        evs[2].record()
        api.pa_decode(q, wl.k_cache, wl.v_cache, st["tables"], st["lens"], max_context_len=wl.max_c, out=out,
                      partition_size=wl.P, workspace=wl.workspace)
        evs[3].record()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    clocks = ClockSampler(local_rank)
    for i in range(Wm):
        device_step(traj[i % n_traj])
    torch.cuda.synchronize()
    assert api.workspace_error(wl.workspace) == 0, "decode reported an error"
    step_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record()
    for i in range(K):
        step_evs[i][0].record()
        device_step(traj[i % n_traj])
        step_evs[i][1].record()
    stop.record()
    torch.cuda.synchronize()
    barrier()
    clocks.mark(t_wall0, time.time())
    total_ms = start.elapsed_time(stop)
    step_times = sorted(e[0].elapsed_time(e[1]) for e in step_evs)

    # the same K steps as separate calls: per-call times, and the decode call's roofline
    for i in range(Wm):
        separate_calls(traj[i % n_traj], [torch.cuda.Event(enable_timing=True) for _ in range(4)])
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(K):
        separate_calls(traj[i % n_traj], evs[i])
    torch.cuda.synchronize()
    barrier()
    clocks.mark(t_wall0, time.time())
    separate_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in evs)
    copy_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    write_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    decode_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    step_bytes = statistics.mean(traj[i % n_traj]["step_bytes"] for i in range(K))
    decode_bytes = statistics.mean(traj[i % n_traj]["decode_bytes"] for i in range(K))
    touched_bytes = round(statistics.mean(wl.touched_bytes(traj[i % n_traj]["lens_host"]) for i in range(n_traj)))
    kv_bytes = statistics.mean(traj[i % n_traj]["kv_bytes"] for i in range(K))
    copy_bytes = statistics.mean(traj[i % n_traj]["n_pairs"] * 2 * Hk * wl.B * d * wl.es * 2 for i in range(K))
    write_bytes = 2 * (S * Hk * d * wl.es * 2) + 8 * S
    n_pairs = statistics.mean(st["n_pairs"] for st in traj)
    lens = traj[0]["lens"].cpu()
    launches_total = sum(launches[i % n_traj] for i in range(K))

    # ---- end to end through the API: captured steps replayed from pinned host memory ----
    # E2E_DEPTH captured steps (sets of buffers) launched in turn with launch_async: the host block
    # manager prepares step i while the GPU runs the steps before it; step i's input copy and the
    # previous steps' output copies run on copy streams beside the kernels.  A step's buffers are
    # refilled only after its previous output has come back (wait()).
    steps = [api.DecodeStep(wl.k_cache, wl.v_cache, S, H, wl.max_blocks, wl.max_c, max_pairs=S,
                            out_dtype=wl.dtype, partition_size=wl.P) for _ in range(E2E_DEPTH)]
    for st in steps:
        st.h_query.copy_(q.cpu())
        st.h_key.copy_(key.cpu())
        st.h_value.copy_(val.cpu())
    es, B = wl.es, wl.B
    e2e_bytes = 0
    stream = torch.cuda.current_stream()

    host_s = []

    def prepare(st):
        nonlocal e2e_bytes
        t_host = time.perf_counter()
        _, pr, _, ln = wl.host_step(st.h_slots, None, st.h_tables, st.h_lens)
        host_s.append(time.perf_counter() - t_host)
        st.set_pairs(pr)
        c_sum, nb_sum = int(ln.sum()), int(((ln + (B - 1)) // B).sum())
        e2e_bytes += (c_sum * Hk * d * 2 * es + S * H * d * es * 2 + 4 * nb_sum + 4 * S
                      + 2 * (S * Hk * d * es * 2) + 8 * S + pr.shape[0] * 2 * (Hk * B * d * es) * 2)

    host_busy = {"prepare": [], "launch": [], "wait": []}   # host seconds per step, by phase

    def e2e_run(n):
        for i in range(n):
            st = steps[i % E2E_DEPTH]
            t0 = time.perf_counter()
            if i >= E2E_DEPTH:
                st.wait()                # step i-E2E_DEPTH's output is in st.h_out; its buffers are free
            t1 = time.perf_counter()
            prepare(st)                  # overlaps the GPU running the previous steps
            t2 = time.perf_counter()
            st.launch_async(stream)
            t3 = time.perf_counter()
            host_busy["wait"].append(t1 - t0)
            host_busy["prepare"].append(t2 - t1)
            host_busy["launch"].append(t3 - t2)
        for st in steps[:min(n, E2E_DEPTH)]:
            st.wait()
        stream.synchronize()

    e2e_run(2)  # warm-up (also grows every sequence by two tokens)
    e2e_bytes = 0
    host_s.clear()
    for v in host_busy.values():
        v.clear()
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    e2e_run(e2e_steps)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    clocks.mark(t_wall0, time.time())
    h2d, d2h = steps[0].h2d_bytes * e2e_steps, steps[0].d2h_bytes * e2e_steps
    e2e_ms = e0.elapsed_time(e1)
    clock_info = clocks.finish()

    total_ms, e2e_ms, decode_ms, copy_ms, write_ms, separate_ms = reduce_max(
        [total_ms, e2e_ms, decode_ms, copy_ms, write_ms, separate_ms], world, dev)
    if rank != 0:
        return None

    peak, peak_kind = load_peaks()
    uniq_bytes = wl.unique_kv_bytes(traj[0]["tables"].cpu(), lens) if hasattr(wl, "unique_kv_bytes") else None
    value = aggregate_value(step_bytes, K, world, total_ms)
    achieved = decode_bytes / (decode_ms * 1e-3) / 1e9
    ms_per_step = total_ms / K
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": round(ms_per_step, 5),
        "step_ms_spread": {"min": round(step_times[0], 5), "median": round(statistics.median(step_times), 5),
                           "max": round(step_times[-1], 5), "of": len(step_times),
                           "note": "CUDA events around each timed step (one pa_decode_step call)"},
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[wl.dtype],
        "data": "synthetic",
        "config": {
            "workload": wl.cfg["desc"],
            "global_batch": S * world,
            "seq_len": f"mean {statistics.mean(lens.tolist()):.0f}, max {max(lens.tolist())}",
            "parallelism": f"replicas x{world} (sequence-sharded, no collective)",
            "partition_size": wl.P,
            "l2": (f"inputs larger than L2: {kv_bytes / 1e9:.2f} GB of K/V read per step"
                   + (f" ({uniq_bytes / 1e9:.2f} GB in distinct blocks: blocks shared by several sequences are "
                      f"read once per sequence, partly from L2)" if uniq_bytes is not None else "") + ", no flush"
                   if (uniq_bytes if uniq_bytes is not None else kv_bytes) > L2_BYTES else
                   f"warm: the {kv_bytes / 1e6:.1f} MB of K/V read per step fit in L2 (no flush)"),
            "step": "host block manager -> pa_decode_step (COW copies, slot writes and the decode plan in one "
                    "kernel, then decode and combine)",
            "step_bytes": round(step_bytes),
            "cow_pairs_per_step": n_pairs,
            "trajectory_steps": n_traj,
            **({"unique_kv_bytes_step0": uniq_bytes,
                "logical_kv_bytes_step0": traj[0]["kv_bytes"]} if uniq_bytes is not None else {}),
        },
        "kernel_ms": {"step": round(ms_per_step, 5), "decode": round(decode_ms, 5),
                      "step_over_decode": round(ms_per_step / decode_ms, 4),
                      "separate_calls": {"copy_blocks": round(copy_ms, 5), "cache_write": round(write_ms, 5),
                                         "decode": round(decode_ms, 5), "step": round(separate_ms, 5)}},
        "kernel_gbs": {"copy_blocks": round(copy_bytes / (copy_ms * 1e-3) / 1e9, 2) if copy_bytes else None,
                       "cache_write": round(write_bytes / (write_ms * 1e-3) / 1e9, 2)},
        "seqs_per_s": round(S * world / (ms_per_step * 1e-3), 1),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "pct_of_nominal_hbm": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "roofline": {
            "bound": "hbm",
            "kernel": "pa_decode (plan + decode_kernel + combine, CUDA events around each of K calls)",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "nominal_gbs": NOMINAL_HBM_GBS,
            "traffic": profiled_traffic(args),
            "algorithmic_bytes_per_launch": decode_bytes,
            "touched_bytes_per_launch": touched_bytes,
            "touched_gbs": round(touched_bytes / (decode_ms * 1e-3) / 1e9, 2),
            "launch_ms": round(decode_ms, 5),
        },
        "clocks": clock_info,
        "e2e": {
            "value": round(world * e2e_bytes / (e2e_ms * 1e-3) / 1e9, 2),
            "unit": "GB/s",
            "h2d_bytes_per_step": h2d // max(e2e_steps, 1),
            "d2h_bytes_per_step": d2h // max(e2e_steps, 1),
            "steps": e2e_steps,
            "ms_per_step": round(e2e_ms / e2e_steps, 5),
            "host_block_manager_ms": round(1e3 * statistics.median(host_s), 5) if host_s else None,
            "host_ms_per_step": {k: round(1e3 * statistics.mean(v), 5) for k, v in host_busy.items() if v},
            "note": "per step: host block manager (prepared while the GPU runs the previous step), H2D "
                    "of the step's inputs from pinned memory, one replay of the captured kernels "
                    "(pa_decode_step: copies, writes and plan, decode, combine), D2H of o; the copies run on "
                    "copy streams beside the "
                    "neighbouring steps' kernels; every step's output is read back (at most "
                    f"{E2E_DEPTH} steps in flight)",
        },
        "gpu_launches": launches_total,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, lens.tolist(), q, target_s=args.cpu_seconds)
    return line


# ---- the oracle on the host cores -----------------------------------------------------------------

def _compact(wl, sample, q_dev=None, tables=None, lens=None, device_cache=True):
    """CPU copies of the sampled sequences' blocks, with a remapped table."""
    t = tables[sample]
    used = torch.unique(t[t >= 0])
    remap = torch.full((wl.n_blocks,), -1, dtype=torch.int32)
    remap[used] = torch.arange(used.numel(), dtype=torch.int32)
    t2 = torch.where(t >= 0, remap[t.clamp(min=0).long()], t)
    kc = wl.k_cache[used.to(wl.k_cache.device)].cpu()
    vc = wl.v_cache[used.to(wl.v_cache.device)].cpu()
    return q_dev[sample].cpu(), kc, vc, t2, lens[sample]


def cpu_baseline(wl, lens, q, target_s=12.0):
    import oracle

    oracle.build()
    tables, lens_t = wl.mgr.build_block_tables(wl.seqs, wl.max_blocks)
    cores = oracle.hardware_threads()
    order = torch.randperm(wl.S, generator=torch.Generator().manual_seed(5)).tolist()
    # calibrate on two sequences, then size the sample for ~target_s seconds
    probe = order[:2]
    qs, kc, vc, t2, ls = _compact(wl, torch.tensor(probe), q, tables, lens_t)
    t0 = time.perf_counter()
    oracle.decode(qs, kc, vc, t2, ls, n_threads=0)
    dt = max(time.perf_counter() - t0, 1e-3)
    per_tok = dt / max(1, int(ls.sum()))
    n_tok_target = target_s / per_tok
    sample, acc = [], 0
    for s in order:
        if acc >= n_tok_target:
            break
        sample.append(s)
        acc += int(lens_t[s])
    qs, kc, vc, t2, ls = _compact(wl, torch.tensor(sample), q, tables, lens_t)
    passes, t0 = 0, time.perf_counter()
    while True:  # whole passes over the sample until about target_s seconds of oracle work
        oracle.decode(qs, kc, vc, t2, ls, n_threads=0)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or passes >= 1000:
            break
    es, Hk, d, H, B = wl.es, wl.Hk, wl.d, wl.H, wl.B
    c = [int(x) for x in ls]
    byt = passes * (sum(c) * Hk * d * 2 * es + len(c) * H * d * es * 2 + 4 * sum(-(-x // B) for x in c) + 4 * len(c))
    return {"value": round(byt / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} pass(es) over {len(sample)} of {wl.S} sequences ({sum(c)} tokens x {H} heads), "
                      f"decode only, fp64 C++ oracle with {cores} threads, {dt:.1f} s"}


def run_swap(args, rank, world, local_rank):
    """Preemption by swapping: K steps of (swap 512 blocks out to pinned host memory, swap them
    back in), gqa8k-shaped blocks (8 kv heads x 16 tokens x 128 dims, bf16: 64 KiB per block for K
    and V).  The roofline is the host link, measured in the same run as pinned copies of the same
    bytes in each direction."""
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    n_dev, n_host, n_swap, Hk, B, d, dt = 4096, 1024, 512, 8, 16, 128, torch.bfloat16
    gen = torch.Generator(device=dev).manual_seed(11 + rank)
    dk = torch.randn((n_dev, Hk, B, d), generator=gen, device=dev).to(dt)
    dv = torch.randn((n_dev, Hk, B, d), generator=gen, device=dev).to(dt)
    hk = torch.empty((n_host, Hk, B, d), dtype=dt).pin_memory()
    hv = torch.empty((n_host, Hk, B, d), dtype=dt).pin_memory()
    g = torch.Generator().manual_seed(12)
    src = torch.randperm(n_dev, generator=g)[:n_swap]
    out_pairs = torch.stack([src, torch.randperm(n_host, generator=g)[:n_swap]], 1).to(torch.int32).to(dev)
    back = torch.randperm(n_dev, generator=g)[:n_swap]
    in_pairs = torch.stack([out_pairs[:, 1].cpu(), back], 1).to(torch.int32).to(dev)
    blk_bytes = Hk * B * d * 2
    moved = 2 * n_swap * blk_bytes * 2          # K and V, out and in
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def step():
        api.pa_swap_blocks(hk, hv, dk, dv, out_pairs)
        api.pa_swap_blocks(dk, dv, hk, hv, in_pairs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    t0 = time.time()
    ev[0].record()
    for _ in range(args.steps):
        step()
    ev[1].record()
    torch.cuda.synchronize()
    clocks.mark(t0, time.time())
    ms = ev[0].elapsed_time(ev[1])
    # host-link reference: plain pinned copies of the same number of bytes, each direction
    a = torch.empty(n_swap * blk_bytes * 2, dtype=torch.uint8, device=dev)
    h = torch.empty(a.numel(), dtype=torch.uint8).pin_memory()
    for _ in range(3):
        h.copy_(a, non_blocking=True)
        a.copy_(h, non_blocking=True)
    torch.cuda.synchronize()
    ev[2].record()
    for _ in range(args.steps):
        h.copy_(a, non_blocking=True)
        a.copy_(h, non_blocking=True)
    ev[3].record()
    torch.cuda.synchronize()
    ref_ms = ev[2].elapsed_time(ev[3])
    clock_info = clocks.finish()
    ms, ref_ms = reduce_max([ms, ref_ms], world, dev)
    if rank != 0:
        return None
    value = aggregate_value(moved, args.steps, world, ms)
    peak = aggregate_value(moved, args.steps, world, ref_ms) / world
    return {"metric": "block swap GB/s (device <-> pinned host, out and back in)", "value": round(value, 2),
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"swap {n_swap} blocks of 8x16x128 bf16 out to pinned host memory and back",
                       "step_bytes": moved},
            "roofline": {"bound": "host link", "achieved": round(value / world, 2), "peak": round(peak, 2),
                         "peak_kind": "pinned torch copies of the same bytes, same run", "unit": "GB/s",
                         "frac": round(value / world / peak, 4), "traffic": None},
            "clocks": clock_info, "gpu_launches": 2 * args.steps}


def run_prefill(args, rank, world, local_rank):
    """Mixed batch through pa_prefill: 16 prompt chunks of 512 tokens at the end of contexts
    U[1024, 4096] plus 64 decode tokens with lognormal contexts (median 1024), GQA 32/8, d 128,
    B 16, bf16.  FLOPs = 4 d (p + 1) per (query token, head) at position p (q.k and p.v of the
    causal prefix); compared with the measured dense bf16 tensor peak."""
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    H, Hk, d, B, dt = 32, 8, 128, 16, torch.bfloat16
    g = W.generator(21 + rank)
    ctx_p = W.lens_uniform(g, 16, 1024, 4096).tolist()
    ctx_d = W.lens_lognormal(g, 64, 1024.0, 1.0, 16, 8192).tolist()
    ctx = ctx_p + ctx_d
    nq = [512] * 16 + [1] * 64
    case = W.paged_case("prefill", ctx, H, Hk, d, B, dt, 21 + rank, sentinel="none", device=dev)
    q_start = torch.tensor([0] + list(torch.tensor(nq).cumsum(0)), dtype=torch.int32, device=dev)
    q = torch.randn((int(q_start[-1]), H, d), generator=torch.Generator(device=dev).manual_seed(5), device=dev).to(dt)
    max_c, max_q = max(ctx), max(nq)
    ws = torch.empty(api.prefill_workspace_size(len(ctx), H, Hk, d, max_c, max_q), dtype=torch.uint8,
                     device=dev)
    out = torch.empty_like(q)
    flops = sum(4 * d * H * sum(c - n + i + 1 for i in range(n)) for c, n in zip(ctx, nq))
    kv_bytes = sum(ctx) * Hk * d * 2 * 2

    def step():
        api.pa_prefill(q, q_start, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                       max_context_len=max_c, max_q_len=max_q, out=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert api.workspace_error(ws) == 0
    clocks = ClockSampler(local_rank)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks.mark(t0, time.time())
    ms = e0.elapsed_time(e1)
    clock_info = clocks.finish()
    (ms,) = reduce_max([ms], world, dev)
    if rank != 0:
        return None
    tflops = world * flops * args.steps / (ms * 1e-3) / 1e12
    # the launches run back to back for about a second under the power cap: the sustained figure
    # is the denominator, the burst one is reported beside it
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        peak, burst = float(peaks["bf16_tflops_sustained"]), float(peaks["bf16_tflops"])
        kind = "measured (MEASURED_PEAKS.json bf16_tflops_sustained, cuBLAS back to back for 4 s)"
    except Exception:
        peak, burst, kind = 1400.0, 1590.0, "fallback (sustained)"
    return {"metric": "paged prefill + decode attention TFLOP/s (mixed batch)", "value": round(tflops, 2),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "16 prompt chunks of 512 tokens (contexts U[1024,4096]) + 64 decode tokens "
                                   "(lognormal contexts), 32/8 heads, d 128, B 16",
                       "flops_per_step": flops, "unique_kv_bytes": kv_bytes},
            "kv_gbs_unique": round(world * kv_bytes * args.steps / (ms * 1e-3) / 1e9, 2),
            "roofline": {"bound": "tensor", "achieved": round(tflops / world, 2), "peak": peak, "peak_kind": kind,
                         "unit": "TFLOP/s", "frac": round(tflops / world / peak, 4),
                         "kernel": "pa_prefill (prefill_umma_kernel dominant), CUDA events around each of K calls",
                         "traffic": profiled_traffic(args),
                         "peak_burst": burst, "frac_of_burst": round(tflops / world / burst, 4)},
            # per call: prefill_plan_kernel and prefill_umma_kernel for the prompt chunks, then
            # plan_kernel, decode_kernel and combine_kernel for the one-token rows
            "clocks": clock_info, "gpu_launches": 5 * args.steps}


def run_cache_ops(args, rank, world, local_rank):
    """The copy-on-write copy and the slot-mapped write at sizes where they are bandwidth-bound:
    4096 (src, dst) pairs of gqa8k-shaped blocks (8 kv heads x 16 tokens x 128 dims, bf16; 256 MiB
    written, twice the L2, so the copies' writes reach DRAM within the launch) and 65536 new tokens
    written through a random slot mapping into a 16384-block pool (1 GiB of K and V)."""
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    n_blocks, Hk, B, d, dt = 16384, 8, 16, 128, torch.bfloat16
    gen = torch.Generator(device=dev).manual_seed(31 + rank)
    kc = torch.randn((n_blocks, Hk, B, d), generator=gen, device=dev).to(dt)
    vc = torch.randn((n_blocks, Hk, B, d), generator=gen, device=dev).to(dt)
    g = torch.Generator().manual_seed(32)
    perm = torch.randperm(n_blocks, generator=g)
    n_pairs = 4096
    pairs = torch.stack([perm[:n_pairs], perm[n_pairs:2 * n_pairs]], 1).to(torch.int32).to(dev)
    T = 65536
    slots = torch.randperm(n_blocks * B, generator=g)[:T].to(dev)
    key = torch.randn((T, Hk, d), generator=gen, device=dev).to(dt)
    val = torch.randn((T, Hk, d), generator=gen, device=dev).to(dt)
    copy_bytes = n_pairs * 2 * (Hk * B * d * 2) * 2
    write_bytes = 2 * (T * Hk * d * 2 * 2) + 8 * T
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for _ in range(args.warmup):
        api.pa_copy_blocks(kc, vc, pairs)
        api.pa_cache_write(kc, vc, key, val, slots)
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    t0 = time.time()
    ev[0].record()
    for _ in range(args.steps):
        api.pa_copy_blocks(kc, vc, pairs)
    ev[1].record()
    for _ in range(args.steps):
        api.pa_cache_write(kc, vc, key, val, slots)
    ev[2].record()
    torch.cuda.synchronize()
    clocks.mark(t0, time.time())
    copy_ms, write_ms = ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])
    clock_info = clocks.finish()
    copy_ms, write_ms = reduce_max([copy_ms, write_ms], world, dev)
    if rank != 0:
        return None
    peak, kind = load_peaks()
    copy_gbs = aggregate_value(copy_bytes, args.steps, world, copy_ms)
    write_gbs = aggregate_value(write_bytes, args.steps, world, write_ms)
    value = aggregate_value(copy_bytes + write_bytes, args.steps, world, copy_ms + write_ms)
    return {"metric": "COW block copy + slot-mapped cache write effective GB/s", "value": round(value, 2),
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round((copy_ms + write_ms) / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{n_pairs} COW pairs of 8x16x128 bf16 blocks + 65536 slot writes (8x128 bf16 K and V)",
                       "copy_bytes": copy_bytes, "write_bytes": write_bytes},
            "kernels": {"copy_blocks": {"GB/s": round(copy_gbs, 2), "frac": round(copy_gbs / world / peak, 4),
                                        "ms": round(copy_ms / args.steps, 5)},
                        "cache_write": {"GB/s": round(write_gbs, 2), "frac": round(write_gbs / world / peak, 4),
                                        "ms": round(write_ms / args.steps, 5)}},
            "roofline": {"bound": "hbm", "achieved": round(value / world, 2), "peak": peak, "peak_kind": kind,
                         "unit": "GB/s", "frac": round(value / world / peak, 4), "traffic": None},
            "clocks": clock_info, "gpu_launches": 2 * args.steps}


def run_reference(args, rank, world):
    """The oracle timed on the host cores, one bounded sample of the workload per step."""
    if rank != 0:
        return None
    import oracle

    oracle.build()
    cfg = dict(WORKLOADS[args.workload])
    if args.block_size:
        cfg["B"] = args.block_size
    if cfg["lens"]:
        lens = cfg["lens"]().tolist()
    else:                                              # shared prefix: prompt + mean tail + the new token
        wl_cls = SharedPrefixPartialWorkload if args.workload == "shared_prefix_partial_bf16" else SharedPrefixWorkload
        lens = [wl_cls.PROMPT + wl_cls.TAIL_MAX // 2 + 1] * cfg["S"]
    S, H, Hk, d, B, dtype = (cfg[k] for k in ("S", "H", "Hk", "d", "B", "dtype"))
    es = torch.finfo(dtype).bits // 8
    cores = oracle.hardware_threads()
    # Per-step sample: a slice of sequences, generated on the CPU with the workload's shapes.
    budget = 100.0 / (args.steps + args.warmup)       # seconds of oracle work per step
    g = torch.Generator().manual_seed(6)

    def make(seqs):
        ls = [lens[s] for s in seqs]
        case = W.paged_case("ref", ls, H, Hk, d, B, dtype, 1234 + seqs[0], sentinel="none", pool_factor=1.0)
        return case

    probe = make([0])
    t0 = time.perf_counter()
    oracle.decode(probe.q, probe.k_cache, probe.v_cache, probe.block_tables, probe.context_lens, n_threads=0)
    per_tok = (time.perf_counter() - t0) / lens[0]
    tok_budget = max(16, int(budget / per_tok))
    # rotate through the sequences; a sequence longer than the budget is cut to the budget
    cases, s = [], 0
    for i in range(min(args.steps + args.warmup, 64)):
        ls = min(lens[s % S], tok_budget)
        case = W.paged_case("ref", [ls], H, Hk, d, B, dtype, 1234 + i, sentinel="none", pool_factor=1.0)
        cases.append(case)
        s += 1
    times, bytes_ = [], []
    for i in range(args.warmup + args.steps):
        c = cases[i % len(cases)]
        t0 = time.perf_counter()
        oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, n_threads=0)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            n = int(c.context_lens.sum())
            bytes_.append(n * Hk * d * 2 * es + c.S * H * d * es * 2 + 4 * (-(-n // B)) + 4 * c.S)
    total = sum(times)
    value = sum(bytes_) / total / 1e9
    sample = (f"each step: one sequence of the workload (cut to <= {tok_budget} tokens), {H} heads, decode only; "
              f"fp64 C++ oracle, {cores} threads")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": cfg["desc"], "global_batch": S, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="pa", choices=["pa", "reference"])
    ap.add_argument("--workload", default="gqa8k_bf16", choices=sorted(WORKLOADS) + ["swap_bf16", "prefill_mixed_bf16", "cache_ops_bf16"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--partition", type=int, default=0, help="decode partition size in tokens (0 = library default)")
    ap.add_argument("--block-size", type=int, default=0, help="tokens per KV block (0 = the workload's own)")
    ap.add_argument("--seqs", type=int, default=0,
                    help="keep only the first N sequences of a decode workload (0 = all; a smaller case for ncu)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        backend = "nccl" if args.impl == "pa" else "gloo"
        if args.impl == "pa":
            torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference" and args.workload in ("swap_bf16", "prefill_mixed_bf16", "cache_ops_bf16"):
            line = {"impl": "reference", "unavailable": "the oracle arm times the decode workloads only"} if rank == 0 else None
        elif args.impl == "reference":
            line = run_reference(args, rank, world)
        elif args.workload == "swap_bf16":
            line = run_swap(args, rank, world, local_rank)
        elif args.workload == "prefill_mixed_bf16":
            line = run_prefill(args, rank, world, local_rank)
        elif args.workload == "cache_ops_bf16":
            line = run_cache_ops(args, rank, world, local_rank)
        else:
            from paged_kv_cache_329_b200 import build

            if rank == 0 and not os.path.exists(os.path.join(ROOT, "paged_kv_cache_329_b200", "libpa.so")):
                build.build()
            if world > 1:
                torch.distributed.barrier()
            line = run_pa(args, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
