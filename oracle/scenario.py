"""Replay a workload on the oracle (TEST INFRASTRUCTURE ONLY).

Runs the workload's block-manager operations on :class:`oracle.BlockManager`,
applies every store and copy-on-write copy to host caches with the oracle's
``store_kv`` / ``copy_blocks``, then evaluates the attention batch with
``paged_attention`` in float64. Only tests, the smoke check and the bench's
CPU-baseline legs use it.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .paged_kv import BlockManager, copy_blocks, paged_attention, store_kv


@dataclass
class OracleRun:
    bm: BlockManager
    k_cache: np.ndarray
    v_cache: np.ndarray
    op_slots: list            # per op: list of slots written (add/append) or []
    op_pairs: list            # per op: list of (src, dst) copy-on-write pairs
    block_tables: np.ndarray  # [S, MB] int32, pad -1
    context_lens: np.ndarray  # [S] int32
    query_start_loc: np.ndarray
    out: np.ndarray | None    # [T, Hq, D] float64


def replay_ops(wl, k_cache, v_cache, bm):
    op_slots, op_pairs = [], []
    for op in wl.ops:
        slots, pairs = [], []
        if op.kind == "add":
            slots = bm.add_seq(op.seq, op.n)
            store_kv(k_cache, v_cache, op.k, op.v, np.asarray(slots, dtype=np.int64))
        elif op.kind == "fork":
            bm.fork(op.parent, op.seq, op.n)
        elif op.kind == "append":
            slots, pairs = bm.append_tokens(op.seq, op.n)
            copy_blocks(k_cache, v_cache, pairs)
            store_kv(k_cache, v_cache, op.k, op.v, np.asarray(slots, dtype=np.int64))
        elif op.kind == "free":
            bm.free_seq(op.seq)
        else:
            raise ValueError(op.kind)
        op_slots.append(list(slots))
        op_pairs.append(list(pairs))
    return op_slots, op_pairs


def run(wl, k_cache: np.ndarray, v_cache: np.ndarray, attention: bool = True) -> OracleRun:
    """Replay ``wl`` on the given initial caches (modified in place)."""
    geo = wl.geometry
    bm = BlockManager(geo.num_blocks, geo.block_size, wl.initial_free_order)
    op_slots, op_pairs = replay_ops(wl, k_cache, v_cache, bm)
    tables, lens = bm.block_table(wl.batch_seqs, geo.max_blocks_per_seq)
    qsl = wl.query_start_loc()
    out = paged_attention(wl.q, k_cache, v_cache, tables, lens, qsl, wl.scale) if attention else None
    return OracleRun(bm, k_cache, v_cache, op_slots, op_pairs, tables, lens, qsl, out)
