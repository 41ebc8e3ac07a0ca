"""Oracle restatement of the paged KV-cache hot path (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may use this module. It shares no code with the CUDA library.

Page legend (titles as published):
  [A] "深入剖析nano-vLLM推理引擎架构：PagedAttention内存管理实现"
  [B] "深入解析 nano-vLLM 推理引擎的分页 KV 缓存与内存优化架构"
  [C] "vLLM核心架构：PagedAttention原理、KV Cache管理、连续批处理机制"

Data model (readings of the pages, each one stated where it is used):
  * The K and V caches are arrays ``[num_blocks, block_size, num_kv_heads,
    head_dim]``; slot ``s`` is row ``s`` of the flat view ``[num_blocks *
    block_size, num_kv_heads * head_dim]``. [B] §"分页 KV 缓存的核心机制" gives
    the cache flattened to slots; the heads axis it drops is kept here.
  * bf16 values are carried as their uint16 bit patterns; fp32 as float32.
  * Every index is a plain Python / NumPy integer; block-table rows are padded
    with -1 and a negative slot means "padding token, write nothing".
"""

from __future__ import annotations

import math
from collections import deque

import numpy as np


# --------------------------------------------------------------------------
# Value decoding (the oracle's own reading of its inputs)
# --------------------------------------------------------------------------

def as_f64(x: np.ndarray) -> np.ndarray:
    """Exact float64 value of a bf16 bit-pattern array (uint16) or a float array.

    A bf16 number is the upper half of an IEEE binary32, so its value is the
    float32 whose bits are ``bits << 16``; converting that to float64 is exact.
    """
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


# --------------------------------------------------------------------------
# Indexing: slot of a logical token position
# --------------------------------------------------------------------------

def slot_of(block_table_row, position: int, block_size: int) -> int:
    """Flat cache slot of logical token ``position`` of one sequence.

    [A] §"PagedAttention：操作系统的内存智慧" and [C] §"一、PagedAttention：虚拟内存的灵感":
    the logical sequence is cut into fixed blocks of ``block_size`` tokens and a
    per-sequence table maps logical block ``position // block_size`` to a
    physical block. Within the block the token keeps its offset, so the slot is
    ``physical_block * block_size + position % block_size``.
    """
    phys = int(block_table_row[position // block_size])
    if phys < 0:
        raise IndexError("logical block %d is unmapped" % (position // block_size))
    return phys * block_size + position % block_size


# --------------------------------------------------------------------------
# a1: slot-mapped KV write
# --------------------------------------------------------------------------

def _flat_rows(cache: np.ndarray) -> np.ndarray:
    nb, bs = cache.shape[0], cache.shape[1]
    return cache.reshape(nb * bs, -1)


def store_kv(k_cache: np.ndarray, v_cache: np.ndarray, k: np.ndarray, v: np.ndarray,
             slot_mapping: np.ndarray) -> None:
    """Write token ``t``'s K and V rows to cache slot ``slot_mapping[t]`` (in place).

    [B] §"分页 KV 缓存的核心机制": the write goes through a per-token
    ``slot_mapping`` into the cache viewed as ``[total_slots, ...]``.
    Reading: a negative slot is a padding token and writes nothing; two tokens
    of one call never share a slot (asserted, the block manager never emits it).
    This is a bit copy: the cache keeps the caller's dtype and bits.
    """
    slots = np.asarray(slot_mapping, dtype=np.int64)
    live = slots >= 0
    sl = slots[live]
    if np.unique(sl).size != sl.size:
        raise ValueError("duplicate slot within one store")
    kf, vf = _flat_rows(k_cache), _flat_rows(v_cache)
    if sl.size and sl.max() >= kf.shape[0]:
        raise IndexError("slot out of range")
    t = k.shape[0]
    kf[sl] = k.reshape(t, kf.shape[1])[live]
    vf[sl] = v.reshape(t, vf.shape[1])[live]


def store_kv_bruteforce(k_cache, v_cache, k, v, slot_mapping) -> None:
    """Same write as :func:`store_kv`, one element at a time in token order."""
    nb, bs, hkv, d = k_cache.shape
    for t in range(k.shape[0]):
        s = int(slot_mapping[t])
        if s < 0:
            continue
        blk, off = s // bs, s % bs
        for h in range(hkv):
            for e in range(d):
                k_cache[blk, off, h, e] = k[t, h, e]
                v_cache[blk, off, h, e] = v[t, h, e]


# --------------------------------------------------------------------------
# a6: copy-on-write block copy
# --------------------------------------------------------------------------

def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, src_dst_pairs) -> None:
    """For each ``(src, dst)`` pair, in order: block ``dst`` := block ``src`` (K and V).

    [C] §"二、KV Cache管理：从浪费到极致复用": a shared page is physically copied
    only when one request writes it (copy-on-write, as in fork). Reading: no
    ``dst`` is ever also a ``src`` and no ``dst`` repeats (asserted), so the
    order of pairs does not matter.
    """
    pairs = np.asarray(src_dst_pairs, dtype=np.int64).reshape(-1, 2)
    if pairs.size:
        dsts = pairs[:, 1]
        if np.unique(dsts).size != dsts.size or np.intersect1d(dsts, pairs[:, 0]).size:
            raise ValueError("chained or repeated copy destinations")
    for src, dst in pairs:
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]


# --------------------------------------------------------------------------
# a3/a5: attention over block tables
# --------------------------------------------------------------------------

def _gather(cache: np.ndarray, table_row, length: int) -> np.ndarray:
    """Keys (or values) ``0..length-1`` of one sequence, all KV heads: ``[L, Hkv, D]``.

    Logical token i is row ``i % bs`` of physical block ``table_row[i // bs]``;
    taking the first ``ceil(L / bs)`` table entries in order and dropping the
    unfilled tail of the last block yields exactly those rows in logical order.
    """
    bs = cache.shape[1]
    n_blk = -(-length // bs)
    blocks = np.asarray(table_row[:n_blk], dtype=np.int64)
    if (blocks < 0).any():
        raise IndexError("unmapped logical block inside the context")
    return cache[blocks].reshape(n_blk * bs, cache.shape[2], cache.shape[3])[:length]


def paged_attention(q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                    scale: float) -> np.ndarray:
    """softmax(q · Kᵀ · scale) · V per query row, keys gathered through the block table.

    Arguments: ``q [T, Hq, D]``; caches ``[NB, bs, Hkv, D]`` (bf16 bits or
    floats); ``block_tables [S, MB]`` (pad -1); ``context_lens [S]``;
    ``query_start_loc [S+1]`` (rows of sequence s are ``qsl[s]..qsl[s+1]-1``).
    Returns float64 ``[T, Hq, D]``.

    Sources: [A] §"PagedAttention：操作系统的内存智慧" and [C]
    §"一、PagedAttention：虚拟内存的灵感" (logical KV of a sequence lives in
    scattered physical blocks found through its table); [B]
    §"工程落地：配置参数与监控指标" (prefill rows and decode rows are both
    attention over that cache). The attention itself is the textbook
    definition; the pages do not write it out.

    Readings: ``context_lens[s]`` counts every key of sequence s, including the
    rows being queried (they are stored first); query row j of a sequence with
    ``q_len`` rows sits at position ``p = L - q_len + j`` and sees keys
    ``0..p``; query head h reads KV head ``h // (Hq / Hkv)``.
    """
    q64 = as_f64(q)
    t_total, hq, d = q64.shape
    hkv = k_cache.shape[2]
    if hq % hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    g = hq // hkv
    out = np.zeros((t_total, hq, d), dtype=np.float64)
    qsl = np.asarray(query_start_loc, dtype=np.int64)
    for s in range(len(context_lens)):
        length = int(context_lens[s])
        r0, r1 = int(qsl[s]), int(qsl[s + 1])
        q_len = r1 - r0
        if q_len == 0:
            continue
        if q_len > length:
            raise ValueError("sequence %d has more query rows than keys" % s)
        # visible[j, i] is True when key i is at or before query position p_j
        pos = length - q_len + np.arange(q_len)
        visible = np.arange(length)[None, :] <= pos[:, None]
        keys_all = as_f64(_gather(k_cache, block_tables[s], length))      # [L, Hkv, D]
        vals_all = as_f64(_gather(v_cache, block_tables[s], length))
        for kvh in range(hkv):
            keys, vals = keys_all[:, kvh, :], vals_all[:, kvh, :]              # [L, D]
            for h in range(kvh * g, (kvh + 1) * g):
                logits = (q64[r0:r1, h, :] @ keys.T) * scale                   # [q_len, L]
                logits = np.where(visible, logits, -np.inf)
                logits = logits - logits.max(axis=1, keepdims=True)
                w = np.exp(logits)
                w = w / w.sum(axis=1, keepdims=True)
                out[r0:r1, h, :] = w @ vals
    return out


def paged_attention_bruteforce(q, k_cache, v_cache, block_tables, context_lens,
                               query_start_loc, scale: float) -> np.ndarray:
    """Same result as :func:`paged_attention` with scalar loops and ``math.exp``.

    For tiny inputs only. Every key is fetched element by element through the
    block table; nothing is vectorised, nothing is max-subtracted beyond the
    explicit running maximum below.
    """
    t_total, hq, d = q.shape
    nb, bs, hkv, _ = k_cache.shape
    g = hq // hkv
    qv = as_f64(q)
    kv = as_f64(k_cache)
    vv = as_f64(v_cache)
    out = np.zeros((t_total, hq, d), dtype=np.float64)
    for s in range(len(context_lens)):
        length = int(context_lens[s])
        r0, r1 = int(query_start_loc[s]), int(query_start_loc[s + 1])
        q_len = r1 - r0
        for j in range(q_len):
            p = length - q_len + j
            for h in range(hq):
                kvh = h // g
                logits = []
                for i in range(p + 1):
                    blk = int(block_tables[s][i // bs])
                    dot = 0.0
                    for e in range(d):
                        dot += float(qv[r0 + j, h, e]) * float(kv[blk, i % bs, kvh, e])
                    logits.append(dot * scale)
                top = max(logits)
                weights = [math.exp(x - top) for x in logits]
                total = sum(weights)
                for e in range(d):
                    acc = 0.0
                    for i in range(p + 1):
                        blk = int(block_tables[s][i // bs])
                        acc += weights[i] * float(vv[blk, i % bs, kvh, e])
                    out[r0 + j, h, e] = acc / total
    return out


# --------------------------------------------------------------------------
# Byte model
# --------------------------------------------------------------------------

def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """K plus V bytes that one token occupies across all layers.

    [C] §"一、PagedAttention：虚拟内存的灵感" works this out for 32 layers, hidden
    size 4096 and FP16: about 1 GB for a 2048-token request.
    """
    return 2 * num_layers * num_kv_heads * head_dim * elem_bytes


# --------------------------------------------------------------------------
# a2: the host block manager
# --------------------------------------------------------------------------

class OutOfBlocks(RuntimeError):
    """The free list holds fewer blocks than the operation needs (state unchanged)."""


class BlockManager:
    """Free list + per-sequence block tables + reference counts + copy-on-write.

    Sources: [A] §"PagedAttention：操作系统的内存智慧" (a list of free physical
    blocks and a per-sequence logical→physical table; a new block is taken from
    the free list only when the current block is full); [A]
    §"连续批处理与内存管理的协同" (a finished request returns all its blocks to the
    free list); [C] §"二、KV Cache管理：从浪费到极致复用" (requests with a common
    prefix point at the same pages, reference counts decide when a page is
    really free, and a shared page is copied only when one of them writes it).

    Readings: the free list is FIFO (allocate from the front, freed blocks go to
    the back) starting from a caller-given order; an operation that needs more
    blocks than are free fails with :class:`OutOfBlocks` and changes nothing;
    a sequence frees its blocks in logical order.
    """

    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None):
        if num_blocks < 0 or block_size <= 0:
            raise ValueError("bad geometry")
        order = list(range(num_blocks)) if initial_free_order is None else [int(b) for b in initial_free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("initial free order must be a permutation of the pool")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

    # -- queries ----------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def refcount(self, block: int) -> int:
        return self.ref[block]

    def seq_len(self, seq_id: int) -> int:
        return self.lens[seq_id]

    def blocks_of(self, seq_id: int) -> list[int]:
        return list(self.tables[seq_id])

    def _blocks_for(self, n_tokens: int) -> int:
        return -(-n_tokens // self.block_size)

    def slot_mapping(self, seq_id: int, start: int, n: int) -> list[int]:
        if start < 0 or n < 0 or start + n > self.lens[seq_id]:
            raise ValueError("positions outside the sequence")
        row = self.tables[seq_id]
        return [slot_of(row, p, self.block_size) for p in range(start, start + n)]

    def block_table(self, seq_ids, max_blocks: int):
        """``([n, max_blocks] int32 table padded with -1, [n] int32 context lengths)``."""
        table = np.full((len(seq_ids), max_blocks), -1, dtype=np.int32)
        lens = np.zeros(len(seq_ids), dtype=np.int32)
        for i, sid in enumerate(seq_ids):
            row = self.tables[sid]
            if len(row) > max_blocks:
                raise ValueError("sequence %d needs more than max_blocks" % sid)
            table[i, :len(row)] = row
            lens[i] = self.lens[sid]
        return table, lens

    # -- mutations --------------------------------------------------------
    def _take(self) -> int:
        b = self.free.popleft()
        self.ref[b] = 1
        return b

    def add_seq(self, seq_id: int, num_tokens: int) -> list[int]:
        """New sequence holding ``num_tokens`` tokens; returns their slots."""
        if seq_id in self.tables or num_tokens < 0:
            raise ValueError("bad add_seq")
        need = self._blocks_for(num_tokens)
        if need > len(self.free):
            raise OutOfBlocks()
        self.tables[seq_id] = [self._take() for _ in range(need)]
        self.lens[seq_id] = num_tokens
        return self.slot_mapping(seq_id, 0, num_tokens)

    def fork(self, parent: int, child: int, num_tokens: int | None = None) -> None:
        """``child`` shares the blocks holding ``parent``'s first ``num_tokens`` tokens."""
        if parent not in self.tables or child in self.tables:
            raise ValueError("bad fork")
        n = self.lens[parent] if num_tokens is None else num_tokens
        if n < 0 or n > self.lens[parent]:
            raise ValueError("bad fork length")
        shared = self.tables[parent][: self._blocks_for(n)]
        for b in shared:
            self.ref[b] += 1
        self.tables[child] = list(shared)
        self.lens[child] = n

    def append_tokens(self, seq_id: int, n: int):
        """Append ``n`` tokens; returns ``(slots, cow_pairs)``.

        If the sequence's last block is partly filled and shared (refcount > 1),
        the first new token triggers copy-on-write: a fresh block replaces it in
        this table, the shared block loses one reference, and ``(old, new)`` is
        returned so the caller copies the block before writing the new rows.
        """
        if seq_id not in self.tables or n < 0:
            raise ValueError("bad append")
        length = self.lens[seq_id]
        row = self.tables[seq_id]
        bs = self.block_size
        cow = n > 0 and length % bs != 0 and self.ref[row[-1]] > 1
        need = self._blocks_for(length + n) - self._blocks_for(length) + (1 if cow else 0)
        if need > len(self.free):
            raise OutOfBlocks()
        pairs = []
        if cow:
            old = row[-1]
            new = self._take()
            self.ref[old] -= 1
            row[-1] = new
            pairs.append((old, new))
        slots = []
        for p in range(length, length + n):
            if p % bs == 0:
                row.append(self._take())
            slots.append(row[p // bs] * bs + p % bs)
        self.lens[seq_id] = length + n
        return slots, pairs

    def free_seq(self, seq_id: int) -> None:
        """Drop one reference to each block of ``seq_id``; blocks reaching 0 go back."""
        if seq_id not in self.tables:
            raise ValueError("unknown sequence")
        for b in self.tables.pop(seq_id):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.lens[seq_id]

    def compact(self) -> list[tuple[int, int]]:
        """Remap every held block into the dense id range ``[0, H)``.

        Source: [A] §"连续批处理与内存管理的协同" lists defragmentation by block
        remapping ("memory compaction") and warns that moving blocks costs
        bandwidth. Readings: H is the number of held blocks; the held blocks
        whose id is H or more, taken in ascending order, move to the free ids
        below H, taken in ascending order; tables and reference counts follow
        their blocks; afterwards the free list is H, H+1, ..., num_blocks-1.
        Returns the ``(src, dst)`` moves; their count is the migration cost.
        """
        held = [b for b in range(self.num_blocks) if self.ref[b] > 0]
        h = len(held)
        movers = [b for b in held if b >= h]
        holes = [b for b in range(h) if self.ref[b] == 0]
        assert len(movers) == len(holes)
        remap = dict(zip(movers, holes))
        for src, dst in remap.items():
            self.ref[dst], self.ref[src] = self.ref[src], 0
        for sid in self.tables:
            self.tables[sid] = [remap.get(b, b) for b in self.tables[sid]]
        self.free = deque(range(h, self.num_blocks))
        return list(zip(movers, holes))

    def cascade_groups(self, seq_ids, min_shared_blocks: int = 1):
        """Runs of consecutive sequences that share leading full blocks.

        Source: [C] §"二、KV Cache管理：从浪费到极致复用" (requests with a common
        prefix point at the same pages, so those pages can be read once for
        all of them). Readings: a group is a run of at least two consecutive
        sequences of the batch; its shared count is the number of leading
        block-table entries identical in every member and full in every member
        (index < length // block_size); runs are taken greedily from the left,
        each as long as its shared count stays >= min_shared_blocks.
        Returns (shared [n] with each member's count and 0 elsewhere,
        groups [(first, count), ...]).
        """
        ids = list(seq_ids)
        n = len(ids)
        rows = [self.tables[s] for s in ids]
        full = [self.lens[s] // self.block_size for s in ids]

        def shared_count(i, j):  # members i .. j-1
            k = 0
            while all(k < full[m] for m in range(i, j)) and all(rows[m][k] == rows[i][k] for m in range(i, j)):
                k += 1
            return k

        shared = [0] * n
        groups = []
        i = 0
        while i < n:
            j = i + 1
            while j < n and shared_count(i, j + 1) >= min_shared_blocks:
                j += 1
            if j - i >= 2:
                c = shared_count(i, j)
                groups.append((i, j - i))
                for m in range(i, j):
                    shared[m] = c
                i = j
            else:
                i += 1
        return shared, groups

    # -- monitoring -------------------------------------------------------
    def stats(self, kv_bytes_per_block: float = 0.0) -> dict:
        """The pool's monitoring figures, from their definitions.

        Source: [A] §"监控与调优要点": block utilisation is allocated blocks over
        all blocks; internal fragmentation is the share of token slots inside
        blocks that hold no token; the mapping-table memory is compared with the
        whole KV cache. The saving from prefix sharing follows [C]
        §"二、KV Cache管理：从浪费到极致复用" (several requests point at the same
        pages).

        Readings: a block is allocated while its reference count is positive; a
        slot is used when some live sequence maps one of its tokens to it (the
        set union over sequences, so a shared slot counts once); the mapping
        table is one int32 physical id per logical block of every sequence; the
        sharing saving is ``1 - physical / logical`` held blocks. Allocation
        latency is a timing of the library's calls and has no oracle value.
        """
        held = [b for b in range(self.num_blocks) if self.ref[b] > 0]
        used = set()
        for sid, row in self.tables.items():
            for p in range(self.lens[sid]):
                used.add(slot_of(row, p, self.block_size))
        logical = sum(len(row) for row in self.tables.values())
        n_held = len(held)
        table_bytes = 4.0 * logical
        return dict(
            num_blocks=self.num_blocks,
            free_blocks=len(self.free),
            held_blocks=n_held,
            num_seqs=len(self.tables),
            logical_blocks=logical,
            tokens=sum(self.lens.values()),
            used_slots=len(used),
            block_utilisation=n_held / self.num_blocks if self.num_blocks else 0.0,
            internal_fragmentation=1.0 - len(used) / (n_held * self.block_size) if n_held else 0.0,
            sharing_saving=1.0 - n_held / logical if logical else 0.0,
            table_bytes=table_bytes,
            table_overhead=(table_bytes / (self.num_blocks * kv_bytes_per_block)
                            if self.num_blocks and kv_bytes_per_block > 0 else 0.0),
        )


def preallocation_fragmentation(lengths, max_len: int) -> float:
    """Unused share of a cache that reserves ``max_len`` token slots per request.

    The contiguous scheme the pages compare against ([C] §"二、KV
    Cache管理：从浪费到极致复用": allocate the maximum length up front): a
    request of ``n`` tokens leaves ``max_len - n`` of its slots empty.
    """
    lengths = [int(n) for n in lengths]
    if not lengths:
        return 0.0
    return 1.0 - sum(lengths) / (len(lengths) * max_len)
