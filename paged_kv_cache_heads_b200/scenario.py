"""Replay a workload through libpa on a CUDA device.

``prepare`` runs the workload's block-manager operations on the library's
block manager (host) and applies every store and copy-on-write copy with the
library's kernels, except the trailing ``step_ops`` operations: their block
manager calls run once to fix slots and copy pairs, and their stores stay
pending in a ``DeviceBatch``. ``run_step`` then performs one pass of the hot
path on that batch: copy-on-write copies, the slot-mapped store of the new
tokens, and attention over the block tables. Re-running it writes the same
bits again, so it can be timed in a loop.

PyTorch only provides device memory and the stream; all work is in libpa.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from . import BlockManager, CacheDesc, PA_BF16, PA_FP32, pa_attention, pa_attention_cascade, \
    pa_attention_cascade_workspace_size, pa_attention_workspace_size, pa_copy_blocks, pa_store_kv
from . import workloads as W


def _to_dev(a: np.ndarray, device) -> torch.Tensor:
    """Upload a host array without reinterpreting its bits (bf16 as int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


def sentinel_cache_dev(geo: W.Geometry, device) -> torch.Tensor:
    shape = (geo.num_blocks, geo.block_size, geo.num_kv_heads, geo.head_dim)
    if geo.dtype == W.BF16:
        return torch.full(shape, int(W.SENTINEL_BF16), dtype=torch.int16, device=device)
    return torch.full(shape, int(W.SENTINEL_FP32), dtype=torch.int32, device=device).view(torch.float32)


def cache_desc(geo: W.Geometry) -> CacheDesc:
    return CacheDesc(geo.num_blocks, geo.block_size, geo.num_kv_heads, geo.head_dim,
                     PA_BF16 if geo.dtype == W.BF16 else PA_FP32)


@dataclass
class DeviceBatch:
    wl: W.Workload
    desc: CacheDesc
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    step_k: torch.Tensor          # [T_step, Hkv, D]
    step_v: torch.Tensor
    step_slots: torch.Tensor      # int32 [T_step]
    step_pairs: torch.Tensor      # int32 [n, 2]
    q: torch.Tensor               # [T, Hq, D]
    out: torch.Tensor
    block_tables: torch.Tensor    # int32 [S, MB]
    context_lens: torch.Tensor    # int32 [S]
    query_start_loc: torch.Tensor # int32 [S+1]
    workspace: torch.Tensor | None
    max_context_len: int
    host: dict = field(default_factory=dict)   # host copies of every index array

    @property
    def num_step_tokens(self) -> int:
        return int(self.step_slots.numel())


def prepare(wl: W.Workload, device="cuda", bm: BlockManager | None = None) -> DeviceBatch:
    geo = wl.geometry
    desc = cache_desc(geo)
    kc = sentinel_cache_dev(geo, device)
    vc = sentinel_cache_dev(geo, device)
    if bm is None:
        bm = BlockManager(geo.num_blocks, geo.block_size, wl.initial_free_order)
    n_setup = len(wl.ops) - wl.step_ops
    op_slots, op_pairs = [], []
    step_k, step_v, step_slots, step_pairs = [], [], [], []
    for i, op in enumerate(wl.ops):
        slots, pairs = [], []
        if op.kind == "add":
            slots = bm.add_seq(op.seq, op.n)
        elif op.kind == "fork":
            bm.fork(op.parent, op.seq, op.n)
        elif op.kind == "append":
            slots, pairs = bm.append_tokens(op.seq, op.n)
        elif op.kind == "free":
            bm.free_seq(op.seq)
        op_slots.append(list(slots))
        op_pairs.append(list(pairs))
        if op.kind not in ("add", "append"):
            continue
        if i < n_setup:
            if pairs:
                p = _to_dev(np.asarray(pairs, dtype=np.int32), device)
                pa_copy_blocks(p, len(pairs), kc, vc, desc)
            if op.n:
                pa_store_kv(_to_dev(op.k, device), _to_dev(op.v, device),
                            _to_dev(np.asarray(slots, dtype=np.int32), device), op.n, kc, vc, desc)
        else:
            step_k.append(op.k)
            step_v.append(op.v)
            step_slots.extend(slots)
            step_pairs.extend(pairs)
    table, lens = bm.block_table(wl.batch_seqs, geo.max_blocks_per_seq)
    qsl = wl.query_start_loc()
    hkv, d = geo.num_kv_heads, geo.head_dim
    npdt = W.numpy_dtype(geo.dtype)
    sk = np.concatenate(step_k) if step_k else np.zeros((0, hkv, d), npdt)
    sv = np.concatenate(step_v) if step_v else np.zeros((0, hkv, d), npdt)
    q = _to_dev(wl.q, device)
    out = torch.zeros_like(q)
    max_ctx = int(lens.max()) if lens.size else 0
    ws_bytes = pa_attention_workspace_size(len(wl.batch_seqs), geo.num_q_heads, wl.max_query_len, max_ctx, desc)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device) if ws_bytes else None
    host = dict(op_slots=op_slots, op_pairs=op_pairs, block_tables=table, context_lens=lens,
                query_start_loc=qsl, step_slots=np.asarray(step_slots, np.int32),
                step_pairs=np.asarray(step_pairs, np.int32).reshape(-1, 2), step_k=sk, step_v=sv,
                bm=bm)
    return DeviceBatch(wl, desc, kc, vc, _to_dev(sk, device), _to_dev(sv, device),
                       _to_dev(host["step_slots"], device), _to_dev(host["step_pairs"], device), q, out,
                       _to_dev(table, device), _to_dev(lens, device), _to_dev(qsl, device), ws, max_ctx, host)


def run_step(b: DeviceBatch, stream=None, attention: bool = True, store: bool = True):
    """One pass of the hot path: CoW copies, new-token store, attention."""
    geo = b.wl.geometry
    if store:
        if b.step_pairs.shape[0]:
            pa_copy_blocks(b.step_pairs, b.step_pairs.shape[0], b.k_cache, b.v_cache, b.desc, stream=stream)
        if b.num_step_tokens:
            pa_store_kv(b.step_k, b.step_v, b.step_slots, b.num_step_tokens, b.k_cache, b.v_cache, b.desc,
                        stream=stream)
    if attention:
        run_attention(b, stream=stream)


def run_attention(b: DeviceBatch, stream=None, out=None):
    geo = b.wl.geometry
    pa_attention(b.q, b.k_cache, b.v_cache, b.block_tables, geo.max_blocks_per_seq, b.context_lens,
                 b.query_start_loc, len(b.wl.batch_seqs), b.wl.num_q_tokens, geo.num_q_heads,
                 b.wl.max_query_len, b.max_context_len, b.wl.scale, b.desc, b.out if out is None else out,
                 b.workspace, stream=stream)


def out_as_f64(t: torch.Tensor, dtype: str) -> np.ndarray:
    """float64 values of an output tensor (bf16 carried as int16 bits)."""
    a = t.detach().cpu().numpy()
    if dtype == W.BF16:
        return W.bf16_bits_to_f32(a.view(np.uint16)).astype(np.float64)
    return a.astype(np.float64)


def cache_bits(t: torch.Tensor) -> np.ndarray:
    a = t.detach().cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a.view(np.uint32)


def capture_step(b: DeviceBatch, pre=None, post=None):
    """Capture one hot-path step (CoW copies, store, attention) in a CUDA graph.

    ``pre`` / ``post`` are optional callables captured before / after the step
    (e.g. host<->device copies of the step's inputs and output). Every libpa
    call in the step is asynchronous, allocates nothing and never synchronises,
    so the whole step can be replayed with one ``graph.replay()``. Run the step
    once eagerly before capturing so one-time set-up (kernel attributes, the
    tensor-map cache) happens outside the capture.
    """
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        if pre is not None:
            pre()
        run_step(b)
        if post is not None:
            post()
    return g


@dataclass
class CascadePlan:
    shared_blocks: torch.Tensor   # int32 [S]
    groups: torch.Tensor          # int32 [G, 2] (first, count)
    num_groups: int
    max_group_size: int
    max_shared_blocks: int
    workspace: torch.Tensor
    host: dict = field(default_factory=dict)


def plan_cascade(b: DeviceBatch, min_shared_blocks: int = 1) -> CascadePlan:
    """Groups of b's batch that share leading blocks (from the library's block
    manager) and a workspace for pa_attention_cascade."""
    shared, groups = b.host["bm"].cascade_groups(b.wl.batch_seqs, min_shared_blocks)
    dev = b.q.device
    ng = int(groups.shape[0])
    mg = int(groups[:, 1].max()) if ng else 0
    ms = int(shared.max()) if shared.size else 0
    ws_bytes = pa_attention_cascade_workspace_size(len(b.wl.batch_seqs), b.wl.geometry.num_q_heads,
                                                   b.max_context_len, ms, b.desc)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    g = torch.from_numpy(np.ascontiguousarray(groups if ng else np.zeros((1, 2), np.int32))).to(dev)
    return CascadePlan(torch.from_numpy(np.ascontiguousarray(shared)).to(dev), g, ng, mg, ms, ws,
                       dict(shared=shared, groups=groups))


def run_attention_cascade(b: DeviceBatch, plan: CascadePlan, stream=None, out=None):
    geo = b.wl.geometry
    pa_attention_cascade(b.q, b.k_cache, b.v_cache, b.block_tables, geo.max_blocks_per_seq, b.context_lens,
                         b.query_start_loc, len(b.wl.batch_seqs), geo.num_q_heads, b.max_context_len,
                         plan.shared_blocks, plan.groups, plan.num_groups, plan.max_group_size,
                         plan.max_shared_blocks, b.wl.scale, b.desc, b.out if out is None else out,
                         plan.workspace, stream=stream)


STEP_INPUTS = ("q", "step_k", "step_v", "step_slots", "step_pairs", "block_tables", "context_lens",
               "query_start_loc")


def pack_step_inputs(b: DeviceBatch):
    """Stage every per-step input in one buffer so that it arrives with a single copy.

    Returns ``(host, dev)``: a pinned host buffer and a device buffer with the
    same layout (each input at a 256-byte aligned offset). The batch's input
    tensors become views of ``dev``, so the library reads them in place; a
    serving loop writes the next step's inputs into ``host`` and issues one
    ``dev.copy_(host, non_blocking=True)``.
    """
    layout, total = [], 0
    for name in STEP_INPUTS:
        t = getattr(b, name)
        nbytes = t.numel() * t.element_size()
        layout.append((name, total, nbytes))
        total += (nbytes + 255) // 256 * 256
    dev = torch.empty(max(total, 256), dtype=torch.uint8, device=b.q.device)
    host = torch.empty(max(total, 256), dtype=torch.uint8).pin_memory()
    for name, off, nbytes in layout:
        t = getattr(b, name)
        view = dev[off:off + nbytes].view(t.dtype).view(t.shape)
        view.copy_(t)
        host[off:off + nbytes].copy_(t.detach().cpu().contiguous().view(-1).view(torch.uint8))
        setattr(b, name, view)
    return host, dev
