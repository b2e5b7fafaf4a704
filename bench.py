#!/usr/bin/env python
"""Paged-decode benchmark: KV-read GB/s and tokens/s on B200, as a fraction of
the HBM roofline.

One step of the decode loop (the whole hot path for one batch):
  host allocator appends one token to every sequence (new block when the last
  one is full, copy-on-write when it is shared) -> pa_copy_blocks for any
  copy-on-write pairs -> pa_reshape_and_cache writes the new tokens' K/V ->
  pa_decode (or pa_decode_split) attends every query head over its sequence.

Default workload: GQA decode, batch 256, 32 q / 8 kv heads, head_dim 128,
block 16, bf16, lognormal context lengths (median 1024, sigma 0.5, cap 8192),
pool 110 % of the blocks in use, synthetic N(0,1) data.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                  [--workload gqa|mha|long] [--kernel decode|split]

Reported line (rank 0):
  value      KV-read GB/s over the K timed steps, inputs resident in HBM
             (per-step allocator outputs are computed before timing), max
             over ranks, whole job (all replicas).  The K steps are captured
             once into a CUDA graph and replayed once in the timed region
             (the same launches without the host's issue cost between them,
             as a serving loop replays its decode step); --eager launches
             them one by one from Python instead.
  e2e        the same metric through the public API with host buffers: the
             live allocator on the host, pinned H2D copies of each step's
             q / new K,V / slots / lengths / copy-on-write pairs, the table
             changes applied on the device (by pa_decode_step itself, or
             pa_update_block_tables when unfused), and a D2H read of the
             step's output, all inside the timed region;
             uploads and downloads run on their own streams through a ring
             of three buffer sets, overlapping the neighbouring steps'
             kernels as a serving loop would.
  other_configs  (default gqa run, 1 GPU) short device-timed runs of the
             mha, gqa at head_dim 64, long-context split and prefix-sharing workloads, each with
             its kernel's roofline fraction.
  roofline   the decode kernel: algorithmic bytes per launch / mean launch
             time (CUDA events on the launching stream) vs measured HBM GB/s.
  cpu_baseline  the fp64 oracle on the host's cores, bounded sample.
Multi-GPU: the decode path is not sharded; N GPUs run N independent replicas
("scaling": "weak"), one process per GPU, timings max-reduced over NCCL.
"""

from __future__ import annotations

import argparse
import datetime
import gc
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import pa_inputs  # noqa: E402

METRIC = "paged decode KV-read GB/s and tokens/s at 1 B200, as fraction of HBM peak"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20
KERNEL_SOURCES = ["paged_kv_cache_359_b200/csrc/decode.cuh",
                  "paged_kv_cache_359_b200/csrc/common.cuh",
                  "paged_kv_cache_359_b200/csrc/launch.cuh"]
TRAFFIC_SUMMARY = "profiles/decode_gqa_b256_traffic.txt"


# --------------------------------------------------------------------------
# ranks
# --------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world, backend):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))


def reduce_scalar(x: float, op: str, world: int, device) -> float:
    """max or sum of a scalar over ranks (identity at world size 1)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    red = torch.distributed.ReduceOp.MAX if op == "max" else torch.distributed.ReduceOp.SUM
    torch.distributed.all_reduce(t, op=red)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# --------------------------------------------------------------------------
# clocks (NVML, sampled in a thread during the timed region)
# --------------------------------------------------------------------------

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            handle = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                handle = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # no NVML: report no clocks rather than guess
            self._nv = None
            self.error = f"nvml unavailable: {e}"

    def sample(self):
        """One reading of the SM clock and the active clock-event reasons."""
        if self._nv is None:
            return
        nv = self._nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for b, name in REASON_BITS.items():
                if bits & b:
                    self.reasons.add(name)
        except Exception as e:
            self.error = str(e)

    def _run(self):
        while not self._stop.is_set() and self.error is None:
            self.sample()
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
               "samples": len(self.samples), "source": "nvml"}
        if self.error:
            out["error"] = self.error
        return out


# --------------------------------------------------------------------------
# workload
# --------------------------------------------------------------------------

def make_problem(name: str, extra_tokens: int, rank: int, block_size=None, head_dim=None):
    if name == "gqa":
        return pa_inputs.gqa(extra_tokens=extra_tokens, block_size=block_size or 16,
                             head_dim=head_dim or 128)
    if name == "mha":
        p = pa_inputs.mha(max_len=2048 + extra_tokens,
                          num_blocks=8192 + 64 * (-(-extra_tokens // 16) + 1))
        return p
    if name == "long":
        p = pa_inputs.long_context()
        # room for the appended tokens
        extra_blocks = 2 * (-(-extra_tokens // 16) + 1)
        nb = p.num_blocks + extra_blocks
        rng = np.random.default_rng(p.seed + 11)
        order = rng.permutation(nb).astype(np.int32)
        max_blocks = p.max_blocks_per_seq + extra_blocks
        tables = pa_inputs.tables_from_order(p.context_lens, order, 16, max_blocks)
        p.num_blocks, p.free_order, p.block_tables = nb, order, tables
        return p
    raise ValueError(f"unknown workload {name}")


def build_prefix_loop(device, extra_tokens: int, kernel: str, partition: int,
                      block_size: int = 16, head_dim: int = 128):
    """64 sequences forked from one (2048 - block_size/2)-token prefix (32 q /
    8 kv heads, bf16), tails U[0, 512]: the parent's prefix is written, the
    children fork it, every sequence appends its tail through the allocator
    (the shared half-full last block is copied on first write), then one
    pa_copy_blocks and one pa_reshape_and_cache fill the cache."""
    import paged_kv_cache_359_b200 as pa
    pp = pa_inputs.prefix(block_size, head_dim, extra_tokens=extra_tokens)
    bs, hk, d, s = pp.block_size, pp.num_kv_heads, pp.head_dim, pp.num_seqs
    cap = pp.max_blocks_per_seq
    alloc = pa.BlockAllocator(pp.num_blocks, bs, pp.free_order)
    tables = np.full((s, cap), -1, dtype=np.int32)
    lens = np.zeros(s, dtype=np.int32)
    pre_slots, _, lens[0] = alloc.extend(tables[0], 0, pp.prefix_len)
    n = -(-pp.prefix_len // bs)
    for i in range(1, s):
        alloc.fork(tables[0], n, tables[i])
        lens[i] = lens[0]
    slots, cows = [], []
    for i in range(s):
        sl, cow, lens[i] = alloc.extend(tables[i], int(lens[i]), int(pp.tail_lens[i]))
        slots.append(sl)
        if cow is not None:
            cows.append(cow)
    dt = pa_inputs.torch_dtype(pp.dtype)
    gen = pa_inputs.generator(device, pp.seed)
    kc = pa_inputs.poisoned_pool(pp.num_blocks, bs, hk, d, dt, gen, device,
                                 np.zeros((pp.num_blocks, bs), bool))
    vc = pa_inputs.poisoned_pool(pp.num_blocks, bs, hk, d, dt, gen, device,
                                 np.zeros((pp.num_blocks, bs), bool))
    pk, pv = pa_inputs.token_rows(pp.prefix_len, hk, d, pp.dtype, pp.seed + 2, device)
    pa.pa_reshape_and_cache(pk, pv, kc, vc, torch.from_numpy(pre_slots).to(device))
    if cows:
        pa.pa_copy_blocks(kc, vc, torch.tensor(cows, dtype=torch.int64, device=device))
    all_slots = np.concatenate(slots) if slots else np.zeros(0, np.int64)
    tk, tv = pa_inputs.token_rows(len(all_slots), hk, d, pp.dtype, pp.seed + 3, device)
    pa.pa_reshape_and_cache(tk, tv, kc, vc, torch.from_numpy(all_slots).to(device))
    q0 = pa_inputs.randn((s, pp.num_heads, d), dt, gen, device)
    torch.cuda.synchronize()
    problem = pa_inputs.PagedProblem(
        name="prefix", num_heads=pp.num_heads, num_kv_heads=hk, head_dim=d, block_size=bs,
        num_blocks=pp.num_blocks, dtype=pp.dtype, context_lens=lens.copy(),
        free_order=pp.free_order, block_tables=tables.copy(), seed=pp.seed, scale=pp.scale)
    loop = DecodeLoop(problem, device, kernel, partition,
                      state=(kc, vc, q0, alloc, tables, lens))
    shared = (pp.prefix_len // bs) * bs            # whole blocks no one has copied
    shared -= shared % 16
    loop.groups = {"starts": torch.tensor([0, s], dtype=torch.int32, device=device),
                   "prefix": torch.tensor([shared], dtype=torch.int32, device=device),
                   "max_size": s, "max_prefix": shared}
    return loop


def unique_kv_bytes(tables: np.ndarray, lens: np.ndarray, problem) -> int:
    """K/V bytes of the distinct physical blocks the batch reads."""
    bs = problem.block_size
    blocks = set()
    for i, n in enumerate(lens):
        blocks.update(tables[i, :-(-int(n) // bs)].tolist())
    return len(blocks) * bs * problem.num_kv_heads * problem.head_dim * 2 * problem.elem_bytes


def decode_kv_bytes(lens: np.ndarray, problem) -> int:
    return int(lens.astype(np.int64).sum()) * problem.num_kv_heads * problem.head_dim * 2 * \
        problem.elem_bytes


def decode_alg_bytes(lens: np.ndarray, problem, fused: bool = False) -> int:
    """K/V rows read + q read + out written + block-table entries + lengths;
    fused: + the new key/value rows read and written into the cache + slots
    (pa_decode_step writes the new block's table entry instead of reading it)."""
    s = len(lens)
    qo = 2 * s * problem.num_heads * problem.head_dim * problem.elem_bytes
    tab = 4 * int(sum(-(-int(x) // problem.block_size) for x in lens)) + 4 * s
    extra = 0
    if fused:
        extra = 2 * 2 * s * problem.num_kv_heads * problem.head_dim * problem.elem_bytes + 8 * s
    return decode_kv_bytes(lens, problem) + qo + tab + extra


def kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic():
    """(DRAM bytes, algorithmic bytes) of the decode launch in the committed
    ncu summary, if it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, TRAFFIC_SUMMARY)
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    if fields.get("kernel_sources_sha256_16") != kernel_hash():
        return None
    try:
        return float(fields["dram_bytes_per_launch"]), float(fields["alg_bytes_of_captured_launch"])
    except (KeyError, ValueError):
        return None


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs: torch copy, read+write)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (earlier measurement on this pool)"


class DecodeLoop:
    """State of one replica's decode loop: cache pool, host allocator, tables."""

    def __init__(self, problem, device, kernel: str, partition: int, state=None):
        import paged_kv_cache_359_b200 as pa
        self.pa = pa
        self.p = problem
        self.device = device
        self.kernel = kernel
        self.partition = partition
        self.ws = None
        self.fused = False
        if state is not None:            # a prebuilt batch (the prefix workload)
            (self.k_cache, self.v_cache, self.q0, self.alloc, self.tables,
             self.lens) = state
            self.out = torch.empty_like(self.q0)
            self.max_len_cap = self.tables.shape[1] * problem.block_size
            return
        data = pa_inputs.materialize(problem, device)
        self.k_cache, self.v_cache = data["k_cache"], data["v_cache"]
        self.q0 = data["q"]
        s, cap = problem.num_seqs, problem.max_blocks_per_seq
        self.alloc = pa.BlockAllocator(problem.num_blocks, problem.block_size, problem.free_order)
        self.tables = np.full((s, cap), -1, dtype=np.int32)
        self.lens = np.zeros(s, dtype=np.int32)
        for i in range(s):
            _, _, ln = self.alloc.extend(self.tables[i], 0, int(problem.context_lens[i]),
                                         want_slots=False)
            self.lens[i] = ln
        n = -(-self.lens // problem.block_size)
        for i in range(s):
            assert (self.tables[i, :n[i]] == problem.block_tables[i, :n[i]]).all()
        self.out = torch.empty_like(self.q0)
        self.ws = None
        self.max_len_cap = cap * problem.block_size

    def workspace(self, max_len):
        need = self.pa.pa_decode_split_workspace_bytes(self.p.num_seqs, self.p.num_heads,
                                                       self.p.head_dim, max_len, self.partition)
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self.ws

    def launches_per_step(self, n_cow: int) -> int:
        per = {"split": 2, "cascade": 2}.get(self.kernel, 1)
        if self.fused:
            return (1 if n_cow else 0) + per
        return (1 if n_cow else 0) + 1 + per

    def prefix_workspace(self):
        need = self.pa.pa_decode_shared_prefix_workspace_bytes(
            self.p.num_seqs, self.p.num_heads, self.p.head_dim, self.groups["max_prefix"])
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self.ws

    def step(self, out, q, key, value, slots_d, tables_d, lens_d, stream=None):
        """The fused step: table update, cache write and decode, in the
        decode's launch(es); ``tables_d`` is updated in place."""
        if self.kernel == "cascade":
            g = self.groups
            self.pa.pa_decode_shared_prefix_step(
                out, q, key, value, self.k_cache, self.v_cache, slots_d, tables_d, lens_d,
                self.p.scale, g["starts"], g["prefix"], g["max_size"], g["max_prefix"],
                self.prefix_workspace(), stream=stream)
        else:
            self.pa.pa_decode_step(out, q, key, value, self.k_cache, self.v_cache, slots_d,
                                   tables_d, lens_d, self.p.scale, stream=stream)

    def decode(self, q, tables_d, lens_d, max_len):
        if self.kernel == "cascade":
            g = self.groups
            self.prefix_workspace()
            self.pa.pa_decode_shared_prefix(self.out, q, self.k_cache, self.v_cache, tables_d,
                                            lens_d, self.p.scale, g["starts"], g["prefix"],
                                            g["max_size"], g["max_prefix"], self.ws)
        elif self.kernel == "split":
            self.pa.pa_decode_split(self.out, q, self.k_cache, self.v_cache, tables_d, lens_d,
                                    self.p.scale, max_len, self.partition, self.workspace(max_len))
        else:
            self.pa.pa_decode(self.out, q, self.k_cache, self.v_cache, tables_d, lens_d,
                              self.p.scale)


def run_device_timed(loop: DecodeLoop, steps: int, warmup: int, world: int, dev_index: int,
                     unique: bool = False, graph: bool = False):
    """Allocator outputs for every step are computed up front and uploaded;
    the timed region holds only device work on inputs resident in HBM.
    graph: the timed steps are captured once into a CUDA graph (after the
    eager warm-up) and the graph is replayed once inside the timed region,
    which runs exactly the same launches without the host's issue cost.
    Events cannot time launches inside a graph, so the decode launches of
    the same steps go into a second graph, replayed after the timed region:
    its time / K is the mean decode launch (back to back; the decode calls
    are idempotent on the final state: the fused step rewrites the same
    rows and table entries, the other decodes only read)."""
    pa, p, dev = loop.pa, loop.p, loop.device
    total = steps + warmup
    slots, cows, tabs, lens = [], [], [], []
    # the fused step keeps one device copy of the tables and updates it itself
    # (pa_decode_step); the other paths take each step's tables as given
    tab_live = torch.from_numpy(loop.tables).to(dev) if loop.fused else None
    for _ in range(total):
        sl, cw = loop.alloc.append_slots(loop.tables, loop.lens)
        slots.append(sl.copy())
        cows.append(cw.astype(np.int64))
        tabs.append(loop.tables.copy())
        lens.append(loop.lens.copy())
    slots_d = torch.from_numpy(np.stack(slots)).to(dev)
    tabs_d = torch.from_numpy(np.stack(tabs)).to(dev)
    lens_d = torch.from_numpy(np.stack(lens)).to(dev)
    cows_d = [torch.from_numpy(c).to(dev) if len(c) else None for c in cows]
    keys, vals, qs = [], [], []
    for st in range(total):
        t = pa_inputs.step_tokens(p.num_seqs, p.num_heads, p.num_kv_heads, p.head_dim, p.dtype,
                                  p.seed, st, dev)
        keys.append(t["key"]); vals.append(t["value"]); qs.append(t["q"])
    max_lens = [int(x.max()) for x in lens]
    stream = torch.cuda.current_stream()
    dec_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]

    def decode_only(i):
        if loop.fused:
            loop.step(loop.out, qs[i], keys[i], vals[i], slots_d[i], tab_live, lens_d[i])
        else:
            loop.decode(qs[i], tabs_d[i], lens_d[i], max_lens[i])

    def step(i, timed_index=None):
        if cows_d[i] is not None:
            pa.pa_copy_blocks(loop.k_cache, loop.v_cache, cows_d[i])
        if not loop.fused:
            pa.pa_reshape_and_cache(keys[i], vals[i], loop.k_cache, loop.v_cache, slots_d[i])
        if timed_index is not None:
            dec_ev[timed_index][0].record()            # the current (or capturing) stream
        if loop.fused:
            loop.step(loop.out, qs[i], keys[i], vals[i], slots_d[i], tab_live, lens_d[i])
        else:
            loop.decode(qs[i], tabs_d[i], lens_d[i], max_lens[i])
        if timed_index is not None:
            dec_ev[timed_index][1].record()

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    g = g_dec = None
    if graph:
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(stream)
        g, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g, stream=cap):
                for j in range(steps):
                    step(warmup + j)
            with torch.cuda.graph(g_dec, stream=cap):
                for j in range(steps):
                    decode_only(warmup + j)
        stream.wait_stream(cap)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev_index) as clocks:
        t0.record(stream)
        if g is not None:
            g.replay()
        else:
            for j in range(steps):
                step(warmup + j, j)
        t1.record(stream)
        clocks.sample()                # the host is ahead: the GPU is still in the region
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    flags = pa.pa_device_error(clear=True)
    if flags:
        raise RuntimeError(f"device error word 0x{flags:x} during the timed region")
    ms = t0.elapsed_time(t1)
    if g_dec is not None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g_dec.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        dec_ms = [e0.elapsed_time(e1) / steps] * steps
        del g, g_dec
    else:
        dec_ms = [a.elapsed_time(b) for a, b in dec_ev]
    timed_lens = lens[warmup:]
    kv = sum(decode_kv_bytes(x, p) for x in timed_lens)
    alg = [decode_alg_bytes(x, p, loop.fused) for x in timed_lens]
    launches = sum(loop.launches_per_step(len(c)) for c in cows[warmup:])
    uniq = (sum(unique_kv_bytes(t, l, p) for t, l in zip(tabs[warmup:], timed_lens))
            if unique else None)
    return {"ms": ms, "kv_bytes": kv, "dec_ms": dec_ms, "dec_alg_bytes": alg, "unique": uniq,
            "launches": launches, "clocks": clocks.summary(),
            "tokens": steps * p.num_seqs,
            "cow_pairs": int(sum(len(c) for c in cows[warmup:]))}


def run_compaction(loop: DecodeLoop, reps: int = 5):
    """Compaction after the timed loop (not part of a step): every other
    sequence ends and is freed, the host allocator packs the live blocks
    below (live + 1 %) blocks, pa_copy_blocks moves their data, the tables
    are remapped, and the survivors decode over the shrunken pool to the same
    output bits as before the move.  The copy is idempotent (its sources are
    not overwritten), so it is repeated ``reps`` times for the timing."""
    pa, p, dev = loop.pa, loop.p, loop.device
    bs = p.block_size
    keep = np.arange(0, p.num_seqs, 2)
    for i in range(1, p.num_seqs, 2):
        loop.alloc.free(loop.tables[i], int(-(-int(loop.lens[i]) // bs)))
    tables, lens = loop.tables[keep].copy(), loop.lens[keep].copy()
    q = loop.q0[torch.from_numpy(keep).to(dev)].contiguous()
    out0 = torch.empty_like(q)
    lens_d = torch.from_numpy(lens).to(dev)
    pa.pa_decode(out0, q, loop.k_cache, loop.v_cache, torch.from_numpy(tables).to(dev), lens_d,
                 p.scale)
    live = sum(1 for r in loop.alloc.ref_counts() if r > 0)
    before = loop.alloc.num_blocks
    target = min(before, live + max(1, live // 100))
    t0 = time.perf_counter()
    moves = loop.alloc.compact(target)
    host_ms = (time.perf_counter() - t0) * 1e3
    n_blocks = (-(-lens // bs)).astype(np.int32)
    t0 = time.perf_counter()
    pa.BlockAllocator.remap_batch(tables, n_blocks, moves)
    remap_ms = (time.perf_counter() - t0) * 1e3
    moves_d = torch.from_numpy(moves.astype(np.int64)).to(dev)
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    pa.pa_copy_blocks(loop.k_cache, loop.v_cache, moves_d)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(reps):
        pa.pa_copy_blocks(loop.k_cache, loop.v_cache, moves_d)
    ev[1].record(stream)
    torch.cuda.synchronize()
    copy_ms = ev[0].elapsed_time(ev[1]) / reps
    out1 = torch.empty_like(q)
    pa.pa_decode(out1, q, loop.k_cache[:target], loop.v_cache[:target],
                 torch.from_numpy(tables).to(dev), lens_d, p.scale)
    torch.cuda.synchronize()
    bits = torch.int16 if out0.element_size() == 2 else torch.int32
    same = bool(torch.equal(out0.view(bits), out1.view(bits)))
    blk = bs * p.num_kv_heads * p.head_dim * 2 * p.elem_bytes       # K and V of one block
    moved = len(moves) * blk
    return {"pool_blocks_before": before, "pool_blocks_after": target, "live_blocks": live,
            "moves": len(moves), "released_gb": round((before - target) * blk / 1e9, 3),
            "host_compact_ms": round(host_ms, 3), "host_remap_ms": round(remap_ms, 3),
            "remapped_tables": int(len(tables)),
            "copy_ms": round(copy_ms, 4),
            "copy_gbs_read_plus_write": round(2 * moved / (copy_ms / 1e3) / 1e9, 1),
            "decode_bits_identical": same}


def _config_entry(loop, res, steps, peak, label, kernel):
    """Kernel and step figures of one short device-timed run."""
    dec_mean_ms = statistics.fmean(res["dec_ms"])
    dec_alg = statistics.fmean(res["dec_alg_bytes"])
    achieved = dec_alg / (dec_mean_ms / 1e3) / 1e9
    step_ms = res["ms"] / steps
    e = {"workload": label, "kernel": kernel, "steps": steps,
         "mean_launch_ms": round(dec_mean_ms, 5), "alg_bytes_per_launch": int(dec_alg),
         "achieved_gbs": round(achieved, 1), "frac": round(achieved / peak, 4),
         "ms_per_step": round(step_ms, 5),
         "value_gbs": round(res["kv_bytes"] / (res["ms"] / 1e3) / 1e9, 1),
         "clocks_sm_mhz": res["clocks"]["sm_mhz"], "clock_reasons": res["clocks"]["reasons"]}
    if res["unique"] is not None:
        # shared prefix blocks are read by every sharer; unique bytes count
        # each physical block once and are the HBM-bound figure
        uniq = res["unique"] / steps
        e["unique_kv_bytes_per_step"] = int(uniq)
        e["unique_gbs"] = round(uniq / (step_ms / 1e3) / 1e9, 1)
        e["frac_unique"] = round(e["unique_gbs"] / peak, 4)
    return e


def run_other_configs(dev, local, peak, steps=10, warmup=3, prefix_steps=64, prefix_warmup=8):
    """The other decode workloads, measured briefly after the headline run:
    MHA batch 64 (pa_decode_step: mapping update, append and decode in one
    launch), the headline's GQA batch at head_dim 64 (pa_decode_step), the
    long-context split at the config's 512-token partitions, and
    the prefix-sharing batch (block 16, head_dim 128) with plain decode
    (pa_decode_step) and with the cascade (pa_decode_shared_prefix_step).
    Each builds its own pool, runs ``warmup`` eager steps and ``steps``
    device-timed steps replayed as one CUDA graph, and is freed.  The prefix
    steps take ~0.03-0.07 ms, so they run ``prefix_steps`` of them: over ten,
    the replay's fixed start and end (~12 us) would add ~4 % to each."""
    out = []

    def run(build, label, kernel, fused=False, unique=False, n=steps, w=warmup):
        loop = build(2 * (n + w) + 4)
        loop.fused = fused
        res = run_device_timed(loop, n, w, 1, local, unique=unique, graph=True)
        out.append(_config_entry(loop, res, n, peak, label, kernel))
        del loop
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        return out[-1]

    run(lambda extra: DecodeLoop(make_problem("mha", extra, 0), dev, "decode", 512),
        "mha_decode_b64", "pa_decode_step", fused=True)
    run(lambda extra: DecodeLoop(make_problem("gqa", extra, 0, None, 64), dev, "decode", 512),
        "gqa_decode_b256_d64", "pa_decode_step", fused=True)
    run(lambda extra: DecodeLoop(make_problem("long", extra, 0), dev, "split", 512),
        "long_context_split_p512", "pa_decode_split")
    plain = run(lambda extra: build_prefix_loop(dev, extra, "decode", 512, 16, 128),
                "prefix_sharing_b64_bs16_d128", "pa_decode_step", fused=True, unique=True,
                n=prefix_steps, w=prefix_warmup)
    casc = run(lambda extra: build_prefix_loop(dev, extra, "cascade", 512, 16, 128),
               "prefix_sharing_b64_bs16_d128", "pa_decode_shared_prefix_step", fused=True,
               unique=True, n=prefix_steps, w=prefix_warmup)
    casc["speedup_vs_pa_decode"] = round(plain["ms_per_step"] / casc["ms_per_step"], 3)
    return out


def _segments(spec):
    """Byte offsets of 256-byte-aligned segments: spec = [(name, nbytes), ...]."""
    off, out = 0, {}
    for name, nbytes in spec:
        out[name] = (off, nbytes)
        off += (nbytes + 255) // 256 * 256
    return out, off


def _view(buf, seg, dtype, shape):
    off, nbytes = seg
    return buf[off:off + nbytes].view(dtype).view(shape)


# untimed steps the end-to-end loop runs after its timed window (see run_e2e)
E2E_TRAIL = 8


def run_e2e(loop: DecodeLoop, steps: int, warmup: int, world: int, ring: int = 4):
    """Through the public API from host buffers, as a serving loop runs it.

    Every step: the host allocator appends a token to every sequence, writing
    the lengths, slots and copy-on-write pairs straight into a pinned
    metadata buffer; the step's inputs go host->device from pinned memory
    (one copy for q and the new K/V rows, one for the metadata); on the
    device pa_copy_blocks runs the copy-on-write pairs, then pa_decode_step
    applies the step's table changes to the device-resident block tables
    (one entry per sequence at most, taken from the slots already uploaded,
    so the table itself never crosses the link), writes the new rows and
    decodes, in one launch (unfused: pa_update_block_tables,
    pa_reshape_and_cache, then the decode); the step's output comes back
    device->host and the host reads it.  A ring of ``ring`` buffer sets lets
    the host run ahead of the last completed download: step i's uploads and
    allocator work are staged, on their own stream, as soon as step i - ring
    has been read back and before step i - 1 is launched, so that when step
    i is launched its upload has usually landed and the compute stream needs
    no dependency on the upload stream; downloads have a third stream, so
    copies overlap the neighbouring steps' kernels.  The timed region spans every copy of
    every timed step.  Python's cyclic garbage collector is paused over it
    (after a collection), as a serving loop does once it has started, so
    that a collection pass does not stall the host in the middle.

    The timed steps are a window of a loop that goes on: two warm-up steps
    lead into it without a pause and E2E_TRAIL untimed steps follow it (t1
    is on the compute stream before their kernels; only their uploads
    overlap the window, which can only lengthen it).  On B200 boxes the last
    steps issued before a loop stops ran up to twice as slow while their
    host-to-device copies were in flight (measured per step with events;
    SM clocks unchanged), an end effect a serving loop does not have."""
    pa, p, dev = loop.pa, loop.p, loop.device
    total = steps + warmup + E2E_TRAIL
    s, cap = loop.tables.shape
    dt = loop.q0.dtype
    esz = loop.q0.element_size()
    bs = p.block_size
    qshape = (s, p.num_heads, p.head_dim)
    kshape = (s, p.num_kv_heads, p.head_dim)
    in_seg, in_bytes = _segments([("q", s * p.num_heads * p.head_dim * esz),
                                  ("k", s * p.num_kv_heads * p.head_dim * esz),
                                  ("v", s * p.num_kv_heads * p.head_dim * esz)])
    meta_seg, meta_bytes = _segments([("lens", s * 4), ("slots", s * 8), ("cows", s * 2 * 8)])
    cow_off = meta_seg["cows"][0]
    host = []
    for st in range(total):
        t = pa_inputs.step_tokens(p.num_seqs, p.num_heads, p.num_kv_heads, p.head_dim, p.dtype,
                                  p.seed + 1, st, "cpu")
        hb = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
        _view(hb, in_seg["q"], dt, qshape).copy_(t["q"])
        _view(hb, in_seg["k"], dt, kshape).copy_(t["key"])
        _view(hb, in_seg["v"], dt, kshape).copy_(t["value"])
        host.append(hb)
    # the allocator works on host tables; the device copy is uploaded once
    # and from then on only updated on the device
    tables_np = loop.tables
    lens_np = loop.lens.copy()
    tables_d = torch.from_numpy(tables_np).to(dev)
    comp = torch.cuda.current_stream()
    up = torch.cuda.Stream(device=dev)      # host -> device
    down = torch.cuda.Stream(device=dev)    # device -> host, so uploads never queue behind it

    class Buf:
        def __init__(self):
            self.inp = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
            self.meta = torch.empty(meta_bytes, dtype=torch.uint8, device=dev)
            self.meta_h = torch.zeros(meta_bytes, dtype=torch.uint8).pin_memory()
            self.q = _view(self.inp, in_seg["q"], dt, qshape)
            self.k = _view(self.inp, in_seg["k"], dt, kshape)
            self.v = _view(self.inp, in_seg["v"], dt, kshape)
            self.lens = _view(self.meta, meta_seg["lens"], torch.int32, (s,))
            self.slots = _view(self.meta, meta_seg["slots"], torch.int64, (s,))
            self.cows = _view(self.meta, meta_seg["cows"], torch.int64, (s, 2))
            self.lens_h = _view(self.meta_h, meta_seg["lens"], torch.int32, (s,)).numpy()
            self.slots_h = _view(self.meta_h, meta_seg["slots"], torch.int64, (s,)).numpy()
            self.cows_h = _view(self.meta_h, meta_seg["cows"], torch.int64, (s, 2)).numpy()
            self.out = torch.empty_like(loop.out)
            self.out_h = torch.empty(tuple(loop.out.shape), dtype=loop.out.dtype).pin_memory()
            self.h2d, self.done, self.d2h = (torch.cuda.Event(), torch.cuda.Event(),
                                             torch.cuda.Event())
            self.used = False
            self.staged = -1                           # the step whose inputs it holds
            self.n = self.meta_used = 0

    bufs = [Buf() for _ in range(ring)]
    counts = {"h2d": 0, "d2h": 0, "kv": 0}
    pairs_h = np.zeros((s, 2), dtype=np.int32)          # copy-on-write pairs of a step

    def read_back(b):
        b.d2h.synchronize()
        float(b.out_h.view(-1)[0])                     # the host reads the result
        b.used = False

    def stage(i):
        """Step i's uploads and host allocator work, one step ahead of its
        launch so that the upload has landed when the launch is issued."""
        b = bufs[i % ring]
        if b.used:
            read_back(b)                               # step i - ring is done with b
        # q and the new rows do not depend on the allocator: their upload goes
        # out first, and the allocator's work overlaps it
        with torch.cuda.stream(up):
            b.inp.copy_(host[i], non_blocking=True)
        # the allocator writes the step's slots straight into the pinned metadata
        _, cw = loop.alloc.append_slots(tables_np, lens_np, slots_out=b.slots_h,
                                        pairs_out=pairs_h)
        b.lens_h[:] = lens_np
        b.n = len(cw)
        if b.n:
            b.cows_h[:b.n] = cw
        b.meta_used = cow_off + 16 * b.n               # lengths, slots, this step's pairs
        with torch.cuda.stream(up):
            b.meta[:b.meta_used].copy_(b.meta_h[:b.meta_used], non_blocking=True)
            b.h2d.record(up)
        b.staged = i

    def launch(i, count):
        b = bufs[i % ring]
        assert b.staged == i
        # an upload that has landed needs no stream dependency
        if not b.h2d.query():
            comp.wait_event(b.h2d)
        if b.n:
            pa.pa_copy_blocks(loop.k_cache, loop.v_cache, b.cows[:b.n], stream=comp)
        if loop.fused:
            # the mapping update, the cache write and the decode, in the
            # decode's launch(es)
            loop.step(b.out, b.q, b.k, b.v, b.slots, tables_d, b.lens, stream=comp)
        else:
            pa.pa_update_block_tables(tables_d, b.lens, b.slots, bs, p.num_blocks, stream=comp)
            pa.pa_reshape_and_cache(b.k, b.v, loop.k_cache, loop.v_cache, b.slots, stream=comp)
            saved_out, loop.out = loop.out, b.out
            with torch.cuda.stream(comp):
                loop.decode(b.q, tables_d, b.lens, int(b.lens_h.max()))
            loop.out = saved_out
        b.done.record(comp)
        with torch.cuda.stream(down):
            down.wait_event(b.done)
            b.out_h.copy_(b.out, non_blocking=True)
            b.d2h.record(down)
        b.used = True
        b.staged = -1
        if count:
            counts["h2d"] += in_bytes + b.meta_used
            counts["d2h"] += b.out_h.numel() * b.out_h.element_size()
            counts["kv"] += decode_kv_bytes(b.lens_h, p)

    def run(lo, hi, count, stage_below):
        """Launch steps lo .. hi - 1, staging each next step (below
        stage_below) before the current one is launched."""
        for i in range(lo, hi):
            if bufs[i % ring].staged != i:
                stage(i)
            if i + 1 < stage_below:
                stage(i + 1)
            launch(i, count)
            next_step[0] = i + 1

    def drain():
        for k in range(ring):                          # oldest first
            b = bufs[(next_step[0] + k) % ring]
            if b.used:
                read_back(b)

    next_step = [0]
    # the last two warm-up steps run after the synchronisation, right before
    # the timed region, so that it opens on a busy GPU (running clocks,
    # active copy links) as in a loop that has been serving for a while; t0
    # follows their kernels on the compute stream and the timed uploads wait
    # for it
    pre = min(2, warmup)
    run(0, warmup - pre, False, warmup - pre)
    drain()
    torch.cuda.synchronize()
    barrier(world)
    gc.collect()
    gc.disable()
    try:
        # the first timed step is staged only after t0
        run(warmup - pre, warmup, False, warmup)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(comp)
        up.wait_event(t0)
        down.wait_event(t0)
        run(warmup, warmup + steps, True, total)
        for b in bufs:
            if b.used:
                comp.wait_event(b.d2h)
        t1.record(comp)
        run(warmup + steps, total, False, total)
    finally:
        gc.enable()
    drain()
    torch.cuda.synchronize()
    barrier(world)
    # the device tables must have followed the host allocator exactly
    n_live = -(-lens_np // bs)
    got = tables_d.cpu().numpy()
    for i in range(s):
        if not (got[i, :n_live[i]] == tables_np[i, :n_live[i]]).all():
            raise RuntimeError(f"device block table of sequence {i} diverged from the host's")
    loop.lens[:] = lens_np
    return {"ms": t0.elapsed_time(t1), "kv_bytes": counts["kv"], "h2d": counts["h2d"] / steps,
            "d2h": counts["d2h"] / steps}


# --------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# --------------------------------------------------------------------------

def oracle_sample_seconds(problem, k_cache, v_cache, q, tables, lens, seqs):
    import oracle
    t = time.perf_counter()
    oracle.paged_decode(q, k_cache, v_cache, tables, lens, problem.scale, seqs=seqs)
    return time.perf_counter() - t


def cpu_baseline(loop: DecodeLoop, budget_s: float = 15.0):
    """The oracle, as it stands, on this host's cores: whole-batch decode
    steps over the current cache until about ``budget_s`` of CPU work."""
    p = loop.p
    kc, vc, q = loop.k_cache.cpu(), loop.v_cache.cpu(), loop.q0.cpu()
    tables, lens = loop.tables.copy(), loop.lens.copy()
    seqs_all = list(range(p.num_seqs))
    done_bytes, done_secs, steps = 0, 0.0, 0
    chunk = max(1, p.num_seqs // 8)
    i = 0
    while done_secs < budget_s and steps < 8 * 8:
        seqs = seqs_all[(i * chunk) % p.num_seqs:][:chunk]
        i += 1
        done_secs += oracle_sample_seconds(p, kc, vc, q, tables, lens, seqs)
        done_bytes += decode_kv_bytes(lens[seqs], p)
        steps += 1
    return {"value": done_bytes / done_secs / 1e9, "unit": "GB/s", "cores": torch.get_num_threads(),
            "kind": "oracle",
            "sample": f"{steps} chunks of {chunk} sequences ({done_secs:.1f} s of fp64 oracle "
                      f"decode over the current cache; host os.cpu_count()={os.cpu_count()})",
            "tokens_per_s": steps * chunk / done_secs}


def run_reference(args, rank, world):
    """--impl reference: the oracle times the same decode loop on the host's
    cores; each step appends one token per sequence (oracle allocator and
    cache write) and decodes a rotating sample of the batch."""
    import oracle
    if world > 1 and rank != 0:
        return
    p = make_problem(args.workload, pool_headroom_tokens(args), 0, args.block_size, args.head_dim)
    data = pa_inputs.materialize(p, "cpu")
    kc, vc = data["k_cache"], data["v_cache"]
    alloc = oracle.BlockAllocator(p.num_blocks, p.block_size, p.free_order)
    tables, lens = [], []
    for x in p.context_lens:
        t = []
        _, _, ln = oracle.extend(alloc, t, 0, int(x))
        tables.append(t)
        lens.append(ln)
    sample = max(1, min(p.num_seqs, args.ref_sample))
    total_bytes, total_s, tokens = 0, 0.0, 0
    for st in range(args.warmup + args.steps):
        new = pa_inputs.step_tokens(p.num_seqs, p.num_heads, p.num_kv_heads, p.head_dim, p.dtype,
                                    p.seed, st, "cpu")
        t0 = time.perf_counter()
        slots, cows = oracle.append_slots(alloc, tables, lens)
        if cows:
            kc, vc = oracle.copy_blocks(kc, vc, cows)
        kc, vc = oracle.reshape_and_cache(new["key"], new["value"], kc, vc, slots)
        seqs = [(st * sample + j) % p.num_seqs for j in range(sample)]
        tab = np.full((p.num_seqs, max(len(t) for t in tables)), -1, dtype=np.int32)
        for i, t in enumerate(tables):
            tab[i, :len(t)] = t
        oracle.paged_decode(new["q"], kc, vc, tab, lens, p.scale, seqs=seqs)
        dt = time.perf_counter() - t0
        if st >= args.warmup:
            total_s += dt
            total_bytes += decode_kv_bytes(np.asarray(lens)[seqs], p)
            tokens += sample
    value = total_bytes / total_s / 1e9
    cores = torch.get_num_threads()
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(p, args),
        "cpu_baseline": {"kind": "oracle", "cores": cores, "value": round(value, 4),
                         "unit": "GB/s",
                         "sample": f"each step: allocator + cache write for all {p.num_seqs} "
                                   f"sequences, fp64 decode of {sample} of them (rotating)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "tokens_per_s": round(tokens / total_s, 2),
    }
    print(json.dumps(line), flush=True)


def pool_headroom_tokens(args) -> int:
    """Tokens each sequence may grow by during a run: the device-timed loop
    and the end-to-end loop each append one per step.  Both bench arms size
    their pool from this, so they run the same configuration."""
    return 2 * (args.steps + args.warmup) + E2E_TRAIL + 4


def workload_config(p, args):
    lens = p.context_lens
    return {"workload": {"gqa": "gqa_decode_b256", "mha": "mha_decode_b64",
                         "long": "long_context_split",
                         "prefix": "prefix_sharing_b64"}[args.workload],
            "num_seqs": p.num_seqs, "num_heads": p.num_heads, "num_kv_heads": p.num_kv_heads,
            "head_dim": p.head_dim, "block_size": p.block_size, "num_blocks": p.num_blocks,
            "context_len_median": int(np.median(lens)), "context_len_max": int(lens.max()),
            "context_tokens": int(lens.astype(np.int64).sum()),
            # internal fragmentation: unused rows of each sequence's last block
            "block_waste_frac": round(1.0 - float(lens.astype(np.int64).sum()) / float(sum(
                -(-int(x) // p.block_size) * p.block_size for x in lens)), 5),
            "kernel": args.kernel + (" step: table update + append fused into the decode"
                                     if args.fused else ""),
            "partition": args.partition,
            "pdl": not getattr(args, "no_pdl", False),
            "timed_steps": "eager launches" if getattr(args, "eager", False)
                           else "one CUDA graph replay",
            "l2": "inputs larger than L2 (KV cache %.2f GB vs 126 MB L2), no flush" %
                  (decode_kv_bytes(lens, p) / 1e9)}


# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["gqa", "mha", "long", "prefix"], default="gqa")
    ap.add_argument("--kernel", choices=["decode", "split", "cascade"], default=None)
    ap.add_argument("--partition", type=int, default=512,
                    help="split kernel partition in tokens (the long-context config's 512; "
                         "4096 measures faster on B200)")
    ap.add_argument("--unfused", action="store_true",
                    help="decode and cascade kernels: pa_reshape_and_cache then pa_decode "
                         "or pa_decode_shared_prefix, instead of pa_decode_step or "
                         "pa_decode_shared_prefix_step (the table update and the cache write "
                         "fused into the decode)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the short runs of the mha, long and prefix workloads that the "
                         "default gqa run appends as other_configs")
    ap.add_argument("--block-size", type=int, default=None,
                    help="gqa / prefix workloads: block size (default 16)")
    ap.add_argument("--head-dim", type=int, default=None,
                    help="gqa / prefix workloads: head_dim (default 128)")
    ap.add_argument("--eager", action="store_true",
                    help="device-timed loop: launch the timed steps one by one from Python "
                         "instead of replaying them as one CUDA graph (the default: the same "
                         "launches without the host's issue cost between them)")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch (PA_OPT_PDL 0)")
    ap.add_argument("--compact", action="store_true",
                    help="after the timed loop: free half the batch, compact the pool, report")
    ap.add_argument("--ref-sample", type=int, default=64,
                    help="sequences decoded per step by the reference arm")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.kernel is None:
        args.kernel = "split" if args.workload == "long" else "decode"
    if args.unfused and args.kernel == "split":
        ap.error("--unfused applies to the decode and cascade kernels (split writes separately)")
    # the decode and cascade kernels' step has the table update and the cache
    # write fused in unless asked otherwise
    args.fused = args.kernel in ("decode", "cascade") and not args.unfused
    if args.compact and args.workload not in ("gqa", "mha"):
        ap.error("--compact runs on the gqa and mha workloads")
    if (args.block_size or args.head_dim) and args.workload not in ("gqa", "prefix"):
        ap.error("--block-size / --head-dim apply to the gqa and prefix workloads")
    if args.kernel == "cascade" and args.workload != "prefix":
        ap.error("--kernel cascade needs the prefix workload (its sequences share a prefix)")
    rank, world, local = dist_env()
    if world != args.gpus and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE {world}")

    if args.impl == "reference":
        if args.workload == "prefix":
            ap.error("the reference arm times the gqa, mha and long workloads")
        dist_init(world, "gloo")
        try:
            run_reference(args, rank, world)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import paged_kv_cache_359_b200 as pa
    pa.pa_set_option("pdl", 0 if args.no_pdl else 1)
    dist_init(world, "nccl")
    try:
        extra = pool_headroom_tokens(args)
        if args.workload == "prefix":
            loop = build_prefix_loop(dev, extra, args.kernel, args.partition,
                                     args.block_size or 16, args.head_dim or 128)
            p = loop.p
        else:
            p = make_problem(args.workload, extra, rank, args.block_size, args.head_dim)
            loop = DecodeLoop(p, dev, args.kernel, args.partition)
        loop.fused = args.fused
        res = run_device_timed(loop, args.steps, args.warmup, world, local,
                               unique=args.workload == "prefix", graph=not args.eager)
        e2e = None if args.no_e2e else run_e2e(loop, args.steps, args.warmup, world)

        ms = reduce_scalar(res["ms"], "max", world, dev)
        kv_all = reduce_scalar(res["kv_bytes"], "sum", world, dev)
        tokens_all = reduce_scalar(res["tokens"], "sum", world, dev)
        secs = ms / 1e3
        value = kv_all / secs / 1e9
        dec_mean_ms = statistics.fmean(res["dec_ms"])
        dec_alg = statistics.fmean(res["dec_alg_bytes"])
        achieved = dec_alg / (dec_mean_ms / 1e3) / 1e9
        peak, peak_src = hbm_peak()
        # the committed capture is of the default gqa decode launch
        default_shape = (args.workload == "gqa" and args.kernel == "decode" and args.fused
                         and args.block_size in (None, 16) and args.head_dim in (None, 128))
        cap = measured_traffic() if default_shape else None
        # scaled from the captured launch to this run's mean launch by
        # algorithmic bytes (DRAM traffic grows with the tokens read)
        traffic = None if cap is None else round(cap[0] * dec_alg / cap[1])
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if p.dtype == "bf16" else "f32",
            "data": "synthetic", "config": workload_config(p, args),
            "tokens_per_s": round(tokens_all / secs, 1),
            "frac_of_nominal_8tbps": round(value / NOMINAL_HBM_GBS, 4),
            "roofline": {"bound": "hbm",
                         "kernel": {"decode": "pa_decode_step" if args.fused else "pa_decode",
                                    "split": "pa_decode_split (partition + reduce)",
                                    "cascade": ("pa_decode_shared_prefix_step" if args.fused else
                                                "pa_decode_shared_prefix") +
                                               " (shared pass, then own tokens merged)"
                                    }[args.kernel],
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_source": peak_src,
                         "frac_of_nominal_8tbps": round(achieved / NOMINAL_HBM_GBS, 4),
                         "traffic": traffic,
                         "alg_bytes_per_launch": int(dec_alg),
                         "mean_launch_ms": round(dec_mean_ms, 5)},
            "gpu_launches": int(reduce_scalar(res["launches"], "sum", world, dev)),
            "clocks": res["clocks"],
            "cow_pairs_timed": res["cow_pairs"],
        }
        if res["unique"] is not None:
            # the shared prefix is read by every sharer: `value` counts each
            # read (logical bytes), unique bytes count each physical block once
            line["unique_kv_gbs"] = round(res["unique"] / secs / 1e9, 2)
            line["unique_kv_bytes_per_step"] = int(res["unique"] / args.steps)
        if e2e is not None:
            e2e_ms = reduce_scalar(e2e["ms"], "max", world, dev)
            e2e_kv = reduce_scalar(e2e["kv_bytes"], "sum", world, dev)
            line["e2e"] = {"value": round(e2e_kv / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                           "h2d_bytes_per_step": int(e2e["h2d"]),
                           "d2h_bytes_per_step": int(e2e["d2h"]),
                           "ms_per_step": round(e2e_ms / args.steps, 4)}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(loop)
        if world == 1 and not args.no_other_configs and default_shape and not args.compact:
            del loop
            torch.cuda.empty_cache()
            line["other_configs"] = run_other_configs(dev, local, peak)
            loop = None
        if args.compact:                     # last: it frees half the batch
            line["compaction"] = run_compaction(loop)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
