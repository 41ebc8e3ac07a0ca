#!/usr/bin/env python
"""Benchmark of the paged KV-cache hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the hot path over one batch: copy-on-write copies (if
the step has any), the slot-mapped store of the step's new tokens, and
attention over the block tables (decode split-K + merge, chunked-prefill rows
when present). Default workload: the Llama-7B-shape decode batch (32
sequences, 32 q = 32 kv heads, head_dim 128, bf16, 16-token blocks, context
lengths U{128..2048}); its ~570 MB of K/V per step is larger than the 126 MB
L2, so no flush is needed between steps.

Prints ONE JSON line on rank 0. ``value`` is query tokens per second over all
ranks (each rank runs its own independent batch: weak scaling, no data-path
collective). ``e2e`` repeats the measurement through the same C-ABI calls
with the step's inputs copied from pinned host memory and the output read
back inside the timed region. ``roofline`` is for the attention call, the
dominant launch. ``--impl reference`` times the CPU oracle instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode-attn query-tokens/s and KV-read HBM GB/s (% of B200 peak)"
UNIT = "query-tokens/s"

# DRAM bytes per attention call from one ncu capture of this workload
# (dram__bytes_read.sum + dram__bytes_write.sum, both attention kernels),
# valid only while the kernel sources are byte-identical to the captured ones.
# DRAM bytes (read + write) of one launch of the workload's decode kernel, from
# `ncu --set full` captures (profiles/), valid while the kernel sources match.
NCU_TRAFFIC = {
    "sources": "14c46f4317e3d7af",   # decode kernel sources of the capture
    "llama7b_decode_b32_bf16": 589856000 + 4239616,    # paged_decode_kernel
    "gqa_long_decode_b16_bf16": 167207680 + 5744640,   # paged_decode_kernel
}


# Every source the decode kernels are compiled from: recorded ncu traffic of a
# decode kernel is used only while these files are unchanged.
DECODE_SOURCES = ("decode.cu", "decode_tc.cu", "decode_common.cuh", "pa_common.cuh", "pa_internal.h",
                  "tcgen05.cuh")


def _sources_digest() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_heads_b200", "csrc")
    for f in DECODE_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    with open(os.path.join(ROOT, "include", "pa.h"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()[:16]


def decode_kernel_name(geo) -> str:
    """The decode kernel libpa runs for this geometry: the CUDA-core kernel,
    unless PA_DECODE_TC=1 selects the tensor-core one (bf16, head_dim 128,
    groups of 2/4/8)."""
    env = os.environ.get("PA_DECODE_TC", "")
    tc = geo.dtype == "bf16" and geo.head_dim == 128 and geo.group in (2, 4, 8) and env == "1"
    return "paged_decode_tc_kernel" if tc else "paged_decode_kernel"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append(dict(sm=float(p[1]), smax=float(p[2]), power=float(p[3]),
                                 hw=p[5], hwt=p[6], swt=p[7], cap=p[8]))
            except ValueError:
                continue
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("cap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        loaded = [r["sm"] for r in rows if r["power"] > 200] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# --------------------------------------------------------------------------
# distributed helpers (also exercised by the CPU gloo tests)
# --------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# --------------------------------------------------------------------------
# algorithmic work of one step
# --------------------------------------------------------------------------

def causal_prefill_flops(L: int, ql: int, head_dim: int, num_q_heads: int) -> int:
    """FLOPs of the prefill rows of one sequence: query row j (absolute
    position L - ql + j) sees L - ql + j + 1 keys, and each (row, key) pair
    costs 2 * head_dim for Q.K and 2 * head_dim for P.V, per query head."""
    pairs = ql * (L - ql) + ql * (ql + 1) // 2   # = sum over j < ql of (L - ql + j + 1)
    return 4 * head_dim * num_q_heads * pairs


def step_work(wl, step_tokens: int, step_pairs: int):
    """Algorithmic bytes / flops of one step, from the workload's sizes only."""
    geo = wl.geometry
    e = 2 if geo.dtype == "bf16" else 4
    row = geo.num_kv_heads * geo.head_dim * e                 # one token's K (or V) row, all heads
    lens = wl.notes["context_lens"]
    attn_kv = attn_qo = prefill_flops = 0
    for L, ql in zip(lens, wl.q_lens):
        if ql == 0:
            continue
        attn_kv += 2 * L * row + 4 * ((L + geo.block_size - 1) // geo.block_size)
        attn_qo += 2 * ql * geo.num_q_heads * geo.head_dim * e
        if ql > 1:
            prefill_flops += causal_prefill_flops(L, ql, geo.head_dim, geo.num_q_heads)
    store = 2 * 2 * step_tokens * row + 4 * step_tokens
    copy = 2 * 2 * step_pairs * geo.block_size * row
    return dict(attn_bytes=attn_kv + attn_qo, attn_kv_bytes=attn_kv, store_bytes=store, copy_bytes=copy,
                prefill_flops=prefill_flops)


def launches_per_step(b) -> int:
    """Kernels one step launches: store, copy (if pairs), decode + split merge,
    prefill + its merge (if q_len > 1)."""
    wl = b.wl
    n = (1 if b.num_step_tokens else 0) + (1 if b.step_pairs.shape[0] else 0) + 2
    if wl.max_query_len > 1:
        n += 2
    return n


# --------------------------------------------------------------------------
# the oracle, timed on the host cores
# --------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [int(p.get("num_threads", 1)) for p in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_setup(wl):
    """Replay everything before the step on the oracle (untimed)."""
    import oracle
    from oracle import scenario as oscen
    from paged_kv_cache_heads_b200 import workloads as W
    geo = wl.geometry
    kc, vc = W.sentinel_cache(geo), W.sentinel_cache(geo)
    bm = oracle.BlockManager(geo.num_blocks, geo.block_size, wl.initial_free_order)
    n_setup = len(wl.ops) - wl.step_ops

    class _Head:
        pass
    head = _Head()
    head.ops = wl.ops[:n_setup]
    oscen.replay_ops(head, kc, vc, bm)
    step = []
    for op in wl.ops[n_setup:]:
        if op.kind == "append":
            slots, pairs = bm.append_tokens(op.seq, op.n)
            step.append((op, np.asarray(slots, np.int64), pairs))
        elif op.kind == "add":
            step.append((op, np.asarray(bm.add_seq(op.seq, op.n), np.int64), []))
    tables, lens = bm.block_table(wl.batch_seqs, geo.max_blocks_per_seq)
    return kc, vc, step, tables, lens


def oracle_step(wl, state):
    import oracle
    kc, vc, step, tables, lens = state
    for op, slots, pairs in step:
        oracle.copy_blocks(kc, vc, pairs)
        oracle.store_kv(kc, vc, op.k, op.v, slots)
    return oracle.paged_attention(wl.q, kc, vc, tables, lens, wl.query_start_loc(), wl.scale)


def time_oracle(wl, budget_s: float = 12.0, min_steps: int = 1, max_steps: int | None = None):
    state = oracle_setup(wl)
    times = []
    t_all = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        oracle_step(wl, state)
        times.append(time.perf_counter() - t0)
        if max_steps is not None and len(times) >= max_steps:
            break
        if len(times) >= min_steps and time.perf_counter() - t_all > budget_s:
            break
    mean = sum(times) / len(times)
    return dict(value=wl.num_q_tokens / mean, unit=UNIT, cores=blas_threads(), kind="oracle",
                sample="%d full steps of %s (store + attention, NumPy float64), %.2f s each"
                       % (len(times), wl.name, mean)), times


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def measure_ours(wl, steps: int, warmup: int, device, gpu_index: int):
    import torch
    import paged_kv_cache_heads_b200 as P
    from paged_kv_cache_heads_b200 import scenario as gs

    P.load_library()
    P.pa_read_device_flags(clear=True)
    b = gs.prepare(wl, device)
    geo = wl.geometry
    # K+V bytes of one block of this single-layer cache: the table's share is that of one layer
    per_block = 2 * geo.block_size * geo.num_kv_heads * geo.head_dim * (2 if geo.dtype == "bf16" else 4)
    bm_stats = b.host["bm"].stats(per_block)
    stream = torch.cuda.current_stream(device)
    for _ in range(max(warmup, 1)):
        gs.run_step(b)
    torch.cuda.synchronize(device)

    # ---- device-resident inputs
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(gpu_index) as clocks:
        torch.cuda.nvtx.range_push("pa_timed")   # lets a profiler select the timed steps only
        start.record(stream)
        for i in range(steps):
            gs.run_step(b, attention=False)
            ev[i][0].record(stream)
            gs.run_attention(b)
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize(device)
    barrier()
    ms_eager = start.elapsed_time(end)
    attn_ms = [a.elapsed_time(z) for a, z in ev]

    # ---- the same device-resident step replayed from a CUDA graph (no host launch gaps)
    # K steps are timed, bracketed by a barrier and a synchronize; the K-step
    # measurement is repeated for about a second so the clock samples cover a
    # long stretch under load, and the median repeat is reported.
    graph = gs.capture_step(b)
    for _ in range(max(warmup, 1)):
        graph.replay()
    torch.cuda.synchronize(device)

    def graph_steps():
        barrier()
        torch.cuda.synchronize(device)
        start.record(stream)
        for _ in range(steps):
            graph.replay()
        end.record(stream)
        torch.cuda.synchronize(device)
        barrier()
        return start.elapsed_time(end)

    with ClockSampler(gpu_index) as clocks_g:
        first = graph_steps()
        repeats = int(min(500, max(1, reduce_max(float(np.ceil(1000.0 / max(first, 1e-3))), device))))
        graph_reps = [first] + [graph_steps() for _ in range(repeats - 1)]
    ms_graph = statistics.median(graph_reps)
    del graph
    ms_total = min(ms_eager, ms_graph)
    if ms_graph <= ms_eager:
        clocks = clocks_g

    # ---- end to end: every step's inputs (q, new K/V rows, slots, CoW pairs,
    # tables, lengths, query starts) staged in one pinned host buffer and sent
    # with one copy; the output read back; the same library calls in between
    host_in, dev_in = gs.pack_step_inputs(b)
    host_out = torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory()
    h2d = host_in.numel() * host_in.element_size()
    d2h = host_out.numel() * host_out.element_size()

    def e2e_step():
        dev_in.copy_(host_in, non_blocking=True)
        gs.run_step(b)
        host_out.copy_(b.out, non_blocking=True)

    for _ in range(max(warmup, 1)):
        e2e_step()
    torch.cuda.synchronize(device)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_eager_ms = e0.elapsed_time(e1)

    # ---- the same e2e step captured once in a CUDA graph (copies in, step, copy out)
    def pre():
        dev_in.copy_(host_in, non_blocking=True)

    graph = gs.capture_step(b, pre=pre, post=lambda: host_out.copy_(b.out, non_blocking=True))
    for _ in range(max(warmup, 1)):
        graph.replay()
    torch.cuda.synchronize(device)
    barrier()
    e0.record(stream)
    for _ in range(steps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_graph_ms = e0.elapsed_time(e1)
    e2e_ms = min(e2e_eager_ms, e2e_graph_ms)
    del graph
    kernels = measure_kernels(b)
    flags = P.pa_read_device_flags(clear=True)
    return dict(bm_stats=bm_stats, kernels=kernels, step_mode="cuda_graph" if ms_graph <= ms_eager else "eager",
                step_eager_ms=ms_eager / steps, step_graph_ms=ms_graph / steps, e2e_eager_ms=e2e_eager_ms, e2e_graph_ms=e2e_graph_ms, ms_total=ms_total, attn_ms=attn_ms, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, clocks=clocks.summary(),
                launches=launches_per_step(b) * steps, timed_repeats=len(graph_reps), step_tokens=b.num_step_tokens,
                step_pairs=int(b.step_pairs.shape[0]), flags=flags, max_context_len=b.max_context_len)


def measure_kernels(b, reps: int = 10):
    """Side measurements of the other kernels on this workload's caches.

    * store_bulk: one pa_store_kv of every cached token of the batch (their
      slots, fresh rows) -- the bandwidth-bound bulk fill;
    * copy: pa_copy_blocks of 256 block pairs (src = a used block, dst = a free one);
    * prefill_only: pa_attention over the sequences with q_len > 1 alone;
    * cascade: pa_attention_cascade on the batch when its sequences share
      leading blocks (bytes actually read: each group's shared blocks once);
    * compaction: the block manager's remap of the held blocks into a dense
      range, and the pa_copy_blocks call that moves their data (last: it
      rewrites the host tables, so nothing runs on this batch afterwards).
    Each is timed with CUDA events over ``reps`` back-to-back calls after a warm-up.
    """
    import torch
    import paged_kv_cache_heads_b200 as P
    from paged_kv_cache_heads_b200 import scenario as gs
    wl, geo = b.wl, b.wl.geometry
    dev = b.k_cache.device
    e = 2 if geo.dtype == "bf16" else 4
    row = geo.num_kv_heads * geo.head_dim * e
    res = {}

    def timed(fn, tag):
        fn()
        torch.cuda.synchronize(dev)
        torch.cuda.nvtx.range_push(tag)  # lets a profiler select these calls
        fn()
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize(dev)
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        z.record()
        torch.cuda.synchronize(dev)
        return a.elapsed_time(z) / reps

    slots = np.concatenate([np.asarray(s, np.int32) for s in b.host["op_slots"] if len(s)])
    n = int(slots.size)
    if n:
        kk = torch.randint(-2000, 2000, (n, geo.num_kv_heads, geo.head_dim), dtype=torch.int16, device=dev) \
            if geo.dtype == "bf16" else torch.randn(n, geo.num_kv_heads, geo.head_dim, device=dev)
        sl = torch.from_numpy(slots).to(dev)
        kc2, vc2 = torch.empty_like(b.k_cache), torch.empty_like(b.v_cache)
        ms = timed(lambda: P.pa_store_kv(kk, kk, sl, n, kc2, vc2, b.desc), "pa_store_bulk")
        by = 4 * n * row + 4 * n
        res["store_bulk"] = {"tokens": n, "launch_ms": ms, "algorithmic_bytes": by, "gbs": by / (ms * 1e-3) / 1e9}
        del kk, kc2, vc2
    used = np.unique(b.host["block_tables"][b.host["block_tables"] >= 0])
    held = set(int(x) for x in used)
    free = [x for x in range(geo.num_blocks) if x not in held][:256]
    npairs = min(len(free), len(used), 256)
    if npairs:
        pairs = torch.from_numpy(np.stack([used[:npairs], np.asarray(free[:npairs])], 1).astype(np.int32)).to(dev)
        ms = timed(lambda: P.pa_copy_blocks(pairs, npairs, b.k_cache, b.v_cache, b.desc), "pa_copy")
        by = 4 * npairs * geo.block_size * row
        res["copy"] = {"pairs": npairs, "launch_ms": ms, "algorithmic_bytes": by, "gbs": by / (ms * 1e-3) / 1e9}
    po = prefill_only_call(b)
    if po is not None:
        fn, flops, npre, t = po
        ms = timed(fn, "pa_prefill_only")
        res["prefill_only"] = {"seqs": npre, "q_tokens": t, "launch_ms": ms, "flops": flops,
                               "tflops": flops / (ms * 1e-3) / 1e12}
    # cascade: when sequences of the batch share leading blocks, the same
    # attention with each group's shared blocks read once
    plan = gs.plan_cascade(b) if all(q == 1 for q in wl.q_lens) else None
    if plan is not None and plan.num_groups:
        out = torch.empty_like(b.out)
        ms = timed(lambda: gs.run_attention_cascade(b, plan, out=out), "pa_cascade")
        shared, groups = plan.host["shared"], plan.host["groups"]
        lens = b.host["context_lens"]
        tok_bytes = 2 * geo.num_kv_heads * geo.head_dim * e
        # keys each sequence reads itself, plus each group's shared blocks once
        own = sum(int(L) - int(sh) * geo.block_size for L, sh in zip(lens, shared))
        once = sum(int(shared[f]) * geo.block_size for f, _ in groups)
        unique = (own + once) * tok_bytes
        logical = int(np.sum(lens)) * tok_bytes
        res["cascade"] = {"groups": int(len(groups)), "shared_blocks": int(plan.max_shared_blocks),
                          "members": int(sum(int(c) for _, c in groups)), "launch_ms": ms,
                          "kv_bytes_read": unique, "kv_bytes_logical": logical,
                          "gbs": unique / (ms * 1e-3) / 1e9, "logical_gbs": logical / (ms * 1e-3) / 1e9}
    # compaction: the block manager remaps every held block into [0, held) and
    # pa_copy_blocks moves their K/V data (repeating the copy is idempotent)
    bm = b.host["bm"]
    held_blocks = bm.num_blocks() - bm.num_free()
    t0 = time.perf_counter()
    moves = bm.compact()
    host_ms = (time.perf_counter() - t0) * 1e3
    if moves:
        dp = torch.tensor(moves, dtype=torch.int32, device=dev)
        ms = timed(lambda: P.pa_copy_blocks(dp, len(moves), b.k_cache, b.v_cache, b.desc), "pa_compact_copy")
        by = 4 * len(moves) * geo.block_size * row
        res["compaction"] = {"moves": len(moves), "held_blocks": held_blocks, "host_remap_ms": host_ms,
                             "launch_ms": ms, "algorithmic_bytes": by, "gbs": by / (ms * 1e-3) / 1e9}
    return res


def prefill_only_call(b):
    """pa_attention over the batch's leading sequences with q_len > 1 alone:
    (call, algorithmic flops, sequences, query tokens), or None."""
    import torch
    import paged_kv_cache_heads_b200 as P
    wl, geo = b.wl, b.wl.geometry
    pre = [i for i, q in enumerate(wl.q_lens) if q > 1]
    if not pre or pre != list(range(len(pre))):
        return None
    dev = b.k_cache.device
    qsl = b.host["query_start_loc"][: len(pre) + 1]
    t = int(qsl[-1])
    lens = b.host["context_lens"][: len(pre)]
    ctx = int(lens.max())
    mq = int(max(wl.q_lens[i] for i in pre))
    ws_b = P.pa_attention_workspace_size(len(pre), geo.num_q_heads, mq, ctx, b.desc)
    ws = torch.empty(max(ws_b, 16), dtype=torch.uint8, device=dev)
    bt, cl, qs = b.block_tables[: len(pre)].contiguous(), b.context_lens[: len(pre)].contiguous(), \
        torch.from_numpy(qsl).to(dev)
    out = torch.empty_like(b.out)
    flops = 0
    for i in pre:
        L, ql = int(lens[i]), wl.q_lens[i]
        flops += causal_prefill_flops(L, ql, geo.head_dim, geo.num_q_heads)

    def fn():
        P.pa_attention(b.q, b.k_cache, b.v_cache, bt, geo.max_blocks_per_seq, cl, qs, len(pre), t,
                       geo.num_q_heads, mq, ctx, wl.scale, b.desc, out, ws, ws_b)
    return fn, flops, len(pre), t


# --------------------------------------------------------------------------
# every configuration: one attention call at a time, L2 flushed before each
# --------------------------------------------------------------------------

SWEEP = ("tiny", "gqa_long", "prefix_cow", "mixed_bs8", "mixed_bs16", "mixed_bs32")
L2_FLUSH_BYTES = 512 << 20   # > 4x the 126 MB L2
L2_BYTES = 126 << 20


def rotated_copies(b, touched_bytes: int):
    """Copies of a prepared batch with their own KV caches, queries and outputs
    (same values), enough that the copies other than the one being called
    hold at least 3x the L2 of the data a call reads, so the called copy's
    data has been evicted since its last use: a cold L2 without the dirty
    lines a flush by writing leaves behind. None when that needs more than 8."""
    import dataclasses
    r = -(-3 * L2_BYTES // max(int(touched_bytes), 1)) + 1
    if r > 8:
        return None
    return [b] + [dataclasses.replace(b, k_cache=b.k_cache.clone(), v_cache=b.v_cache.clone(), q=b.q.clone(),
                                      out=b.out.clone()) for _ in range(max(r, 2) - 1)]


def timed_calls(fn, reps: int, flush=None):
    """Each of ``reps`` calls timed alone with CUDA events on the current
    stream. ``fn`` is one call, or a list of calls on rotated copies of the
    inputs taken in turn (so each call finds its data evicted from L2 by the
    others). Before each call, outside the timed interval: with ``flush`` (two
    buffers of L2_FLUSH_BYTES), a write of the first evicts the L2 and a read
    of the second then evicts the first's dirty lines, so their write-back does
    not land inside the call; without it, a short spin keeps the GPU busy while
    the host enqueues the call, so the interval holds device time only.
    Returns median / p10 / p90 in ms."""
    import torch
    fns = fn if isinstance(fn, (list, tuple)) else [fn]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for f in fns:
        f()
    torch.cuda.synchronize()
    for i in range(reps):
        if flush is not None:
            flush[0].fill_(i & 0x7F)
            flush[2].copy_(flush[1].view(-1, 1 << 16).amax(dim=1))
        else:
            torch.cuda._sleep(200000)
        ev[i][0].record()
        fns[i % len(fns)]()
        ev[i][1].record()
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(z) for a, z in ev)
    return {"median_ms": t[len(t) // 2], "p10_ms": t[len(t) // 10], "p90_ms": t[(9 * len(t)) // 10], "reps": reps}


def measure_config(name: str, hbm_peak: float, bf16_peak: float, flush, reps: int = 30, oracle: bool = True):
    """Attention call of one configuration (L2 cold), its prefill rows alone,
    its cascade call when sequences share a prompt, and one oracle step."""
    import torch
    import paged_kv_cache_heads_b200 as P
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = build_workload(name)
    geo = wl.geometry
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    work = step_work(wl, b.num_step_tokens, int(b.step_pairs.shape[0]))
    copies = rotated_copies(b, work["attn_bytes"])
    if copies is not None:
        t = timed_calls([(lambda c=c: gs.run_attention(c)) for c in copies], reps)
        l2 = "rotated over %d copies of the KV caches, queries and outputs (the others hold >= 3x the L2); " \
             "no flush" % len(copies)
    else:
        t = timed_calls(lambda: gs.run_attention(b), reps, flush)
        l2 = "flushed before each call (%d MB write, then %d MB read)" % (L2_FLUSH_BYTES >> 20, L2_FLUSH_BYTES >> 20)
    ms = t["median_ms"]
    ent = {"attention_us": ms * 1e3, "p10_us": t["p10_ms"] * 1e3, "p90_us": t["p90_ms"] * 1e3, "reps": reps,
           "query_tokens_per_s": wl.num_q_tokens / (ms * 1e-3), "algorithmic_bytes": work["attn_bytes"],
           "gbs": work["attn_bytes"] / (ms * 1e-3) / 1e9,
           "frac_of_hbm_peak": work["attn_bytes"] / (ms * 1e-3) / 1e9 / hbm_peak, "l2": l2}
    e = 2 if geo.dtype == "bf16" else 4
    tok_bytes = 2 * geo.num_kv_heads * geo.head_dim * e
    lens = b.host["context_lens"]
    po = prefill_only_call(b)
    if po is not None:
        fn, flops, npre, qt = po
        tp = timed_calls(fn, reps, flush)
        ent["prefill_only"] = {"seqs": npre, "q_tokens": qt, "flops": flops, "us": tp["median_ms"] * 1e3,
                               "l2": "flushed before each call (%d MB write, then %d MB read)" % (L2_FLUSH_BYTES >> 20, L2_FLUSH_BYTES >> 20),
                               "tflops": flops / (tp["median_ms"] * 1e-3) / 1e12,
                               "frac_of_bf16_peak": flops / (tp["median_ms"] * 1e-3) / 1e12 / bf16_peak}
    plan = gs.plan_cascade(b) if all(q == 1 for q in wl.q_lens) else None
    if plan is not None and plan.num_groups:
        out = torch.empty_like(b.out)
        if copies is not None:
            tc_ = timed_calls([(lambda c=c: gs.run_attention_cascade(c, plan, out=out)) for c in copies], reps)
        else:
            tc_ = timed_calls(lambda: gs.run_attention_cascade(b, plan, out=out), reps, flush)
        shared, groups = plan.host["shared"], plan.host["groups"]
        own = sum(int(L) - int(sh) * geo.block_size for L, sh in zip(lens, shared))
        once = sum(int(shared[f]) * geo.block_size for f, _ in groups)
        unique = (own + once) * tok_bytes
        cms = tc_["median_ms"]
        ent["cascade"] = {"us": cms * 1e3, "kv_bytes_read": unique, "kv_bytes_logical": int(np.sum(lens)) * tok_bytes,
                          "gbs": unique / (cms * 1e-3) / 1e9, "frac_of_hbm_peak": unique / (cms * 1e-3) / 1e9 / hbm_peak}
        # the plain call reads every distinct block from HBM once as well
        # (shared ones are L2 hits after the first read)
        ent["unique_kv_bytes"] = unique
        ent["frac_of_hbm_peak_unique"] = (unique + work["attn_bytes"] - work["attn_kv_bytes"]) / (ms * 1e-3) / 1e9 \
            / hbm_peak
    ent["device_flags"] = P.pa_read_device_flags(clear=True)
    del b, copies
    torch.cuda.empty_cache()
    if oracle:
        cpu, _ = time_oracle(wl, budget_s=0.0, min_steps=1, max_steps=1)
        ent["oracle"] = {"query_tokens_per_s": cpu["value"], "cores": cpu["cores"], "sample": cpu["sample"]}
    return ent


def workload_config(wl, world: int, l2_note: str):
    geo = wl.geometry
    lens = wl.notes["context_lens"]
    return {"workload": wl.name, "num_seqs": len(wl.batch_seqs), "num_q_tokens": wl.num_q_tokens,
            "num_q_heads": geo.num_q_heads, "num_kv_heads": geo.num_kv_heads, "head_dim": geo.head_dim,
            "block_size": geo.block_size, "num_blocks": geo.num_blocks, "kv_dtype": geo.dtype,
            "context_tokens": int(sum(lens)), "max_context_len": int(max(lens)),
            "parallelism": "dp%d (independent replicas)" % world, "l2": l2_note}


PREFILL_SCALING = (4, 16, 64)  # chunks of 256 tokens in the prefill-only scaling sweep


def prefill_scaling(bf16_peak: float, flush, reps: int = 10):
    """Prefill-only calls of n 256-token chunks (the mixed batches' geometry:
    32 q / 8 kv heads, D 128, bf16, block size 16; prior contexts drawn from
    U{0..1792}, seeded), the L2 flushed before each call: how the prefill rate
    grows once the per-CTA fixed costs are spread over more key tiles."""
    import numpy as np
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs, workloads as W
    out = {}
    for n in PREFILL_SCALING:
        ctx = [int(x) for x in np.random.default_rng(7 + n).integers(0, 1793, size=n)]
        wl = W.random_case(900 + n, num_seqs=n, q_lens=[256] * n, ctx_extra=ctx, num_kv_heads=8, group=4,
                           head_dim=128, block_size=16, dtype=W.BF16)
        b = gs.prepare(wl)
        gs.run_step(b)
        torch.cuda.synchronize()
        flops = sum(causal_prefill_flops(c + 256, 256, 128, 32) for c in ctx)
        t = timed_calls(lambda: gs.run_attention(b), reps, flush)
        ms = t["median_ms"]
        out["chunks_%d" % n] = {"us": ms * 1e3, "gflop": flops / 1e9, "tflops": flops / ms / 1e9,
                                "frac_of_bf16_peak": flops / ms / 1e9 / bf16_peak}
        del b
        torch.cuda.empty_cache()
    out["l2"] = "flushed before each call (%d MB write, then %d MB read)" % (L2_FLUSH_BYTES >> 20, L2_FLUSH_BYTES >> 20)
    return out


def build_workload(name: str):
    from paged_kv_cache_heads_b200 import workloads as W
    if name == "prefix_cow_p2000":
        return W.prefix_cow_decode(prefix_len=2000)
    return W.CONFIGS[name]()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama7b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the per-configuration sweep that the default workload adds at N=1")
    args = ap.parse_args()
    world, rank, local = dist_env()
    hbm_peak, bf16_peak, peak_src = measured_peaks()

    if args.impl == "reference":
        if rank != 0:
            return 0
        wl = build_workload(args.workload)
        budget = 60.0
        cpu, times = time_oracle(wl, budget_s=budget, min_steps=args.steps + args.warmup,
                                 max_steps=args.steps + args.warmup)
        timed = times[args.warmup:] or times
        ms = 1e3 * sum(timed) / len(timed)
        value = wl.num_q_tokens / (ms / 1e3)
        cpu["value"] = value
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": len(timed),
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
                "config": workload_config(wl, 1, "host memory (CPU oracle)"), "cpu_baseline": cpu,
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                "gpu_launches": 0}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local

    wl = build_workload(args.workload)
    r = measure_ours(wl, args.steps, args.warmup, device, gpu_index)
    work = step_work(wl, r["step_tokens"], r["step_pairs"])
    ms_step = reduce_max(r["ms_total"], device) / args.steps
    tokens_all = reduce_sum(float(wl.num_q_tokens), device)
    e2e_ms = reduce_max(r["e2e_ms"], device) / args.steps
    attn_ms = statistics.mean(r["attn_ms"])
    achieved = work["attn_bytes"] / (attn_ms * 1e-3) / 1e9
    digest = _sources_digest()
    traffic = NCU_TRAFFIC.get(wl.name) if NCU_TRAFFIC.get("sources") == digest else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, _ = time_oracle(wl, budget_s=12.0)

    # every other configuration, one attention call at a time (N=1 only)
    configs = None
    if world == 1 and args.workload == "llama7b" and not args.no_sweep:
        import torch
        flush = (torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device),
                 torch.ones(L2_FLUSH_BYTES, dtype=torch.uint8, device=device),
                 torch.empty(L2_FLUSH_BYTES >> 16, dtype=torch.uint8, device=device))
        configs = {}
        with ClockSampler(gpu_index) as sweep_clocks:
            for name in SWEEP:
                configs[name] = measure_config(name, hbm_peak, bf16_peak, flush,
                                               oracle=not args.no_cpu_baseline)
            configs["prefill_scaling"] = prefill_scaling(bf16_peak, flush)
        configs["clocks"] = sweep_clocks.summary()
        del flush

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    roof = {"kernel": "pa_attention (%s + decode_combine_kernel%s)"
                      % (decode_kernel_name(wl.geometry), " + paged_prefill_kernel" if wl.max_query_len > 1 else ""),
            "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "traffic": traffic,
            "traffic_source": ("dram__bytes_read.sum + dram__bytes_write.sum of the decode kernel from one ncu "
                               "capture of this workload (profiles/), decode sources digest %s" % digest)
            if traffic is not None else "none: the decode kernel sources differ from the captured ones",
            "peak_source": peak_src + " (MEASURED_PEAKS.json hbm_gbs)"
            if peak_src == "measured" else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_launch": work["attn_bytes"], "launch_ms": attn_ms,
            "kv_read_gbs": work["attn_kv_bytes"] / (attn_ms * 1e-3) / 1e9}
    kern = r["kernels"]
    for k in ("store_bulk", "copy", "compaction", "cascade"):
        if k in kern:
            kern[k]["frac_of_hbm_peak"] = kern[k]["gbs"] / hbm_peak
    if "prefill_only" in kern:
        kern["prefill_only"]["frac_of_bf16_peak"] = kern["prefill_only"]["tflops"] / bf16_peak
        kern["prefill_only"]["peak_tflops"] = bf16_peak
    line = {"metric": METRIC, "value": tokens_all / (ms_step * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.geometry.dtype == "bf16" else "fp32",
            "data": "synthetic (seeded N(0,1) K/V/Q, random-init; no dataset)",
            "config": workload_config(wl, world, "KV read per step %.0f MB > 126 MB L2; no flush"
                                      % (work["attn_kv_bytes"] / 1e6)),
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": tokens_all / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": r["h2d"],
                    "d2h_bytes_per_step": r["d2h"], "ms_per_step": e2e_ms,
                    "mode": "cuda_graph" if r["e2e_graph_ms"] <= r["e2e_eager_ms"] else "eager",
                    "eager_ms_per_step": r["e2e_eager_ms"] / args.steps,
                    "graph_ms_per_step": r["e2e_graph_ms"] / args.steps},
            "step_launch": {"mode": r["step_mode"], "eager_ms_per_step": r["step_eager_ms"],
                            "graph_ms_per_step": r["step_graph_ms"]},
            "gpu_launches": r["launches"] * r["timed_repeats"], "timed_repeats": r["timed_repeats"],
            "clocks": r["clocks"], "device_flags": r["flags"],
            "kernels": kern,
            "block_manager": {k: (round(v, 6) if isinstance(v, float) else v) for k, v in r["bm_stats"].items()},
            "step_bytes": work["attn_bytes"] + work["store_bytes"] + work["copy_bytes"]}
    if configs is not None:
        line["configs"] = configs
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
