"""Seeded synthetic workloads for the paged KV-cache hot path.

This module only draws random numbers and packs them; it holds none of the
method's arithmetic (no slot computation, no block allocation, no attention).
Both the CUDA path and the oracle consume the same ``Workload`` objects.

A workload is a geometry, an initial free-list order (a seeded permutation of
the pool), a list of block-manager operations with the K/V rows each one
stores, and one attention batch (which sequences, how many query rows each,
the query values). Values are drawn as float32 from N(0, 1) and rounded once
to the cache dtype; bf16 travels as uint16 bit patterns.

The five named configurations follow the workloads of the pages' serving
setting: 16-token blocks, a 128-block / 512-block per-sequence cap, batches of
up to 32-64 sequences, 256-token prefill chunks, and a long shared system
prompt; every size and distribution is stated in the builder that makes it.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BF16 = "bf16"
FP32 = "fp32"


# --------------------------------------------------------------------------
# dtype helpers for input generation
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """float32 value of bf16 bit patterns (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def numpy_dtype(dtype: str):
    return np.uint16 if dtype == BF16 else np.float32


def elem_bytes(dtype: str) -> int:
    return 2 if dtype == BF16 else 4


# --------------------------------------------------------------------------
# data model
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class Geometry:
    num_blocks: int
    block_size: int
    num_kv_heads: int
    num_q_heads: int
    head_dim: int
    dtype: str
    max_blocks_per_seq: int

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def row_elems(self) -> int:
        return self.num_kv_heads * self.head_dim


@dataclass
class Op:
    """One block-manager operation.

    kind: "add" (new sequence of n tokens), "fork" (seq shares parent's first n
    tokens), "append" (n more tokens), "free". For "add"/"append" ``k``/``v``
    hold the n new rows ``[n, Hkv, D]`` that the caller stores after the op.
    """
    kind: str
    seq: int
    n: int = 0
    parent: int = -1
    k: np.ndarray | None = None
    v: np.ndarray | None = None


@dataclass
class Workload:
    name: str
    geometry: Geometry
    initial_free_order: np.ndarray            # int32 [num_blocks]
    ops: list[Op]
    batch_seqs: list[int]                     # sequences in the attention batch, in row order
    q_lens: list[int]                         # query rows per batch sequence
    q: np.ndarray                             # [T, Hq, D] (uint16 bits or float32)
    scale: float
    step_ops: int = 0                         # trailing ops that belong to the timed step
    notes: dict = field(default_factory=dict)

    @property
    def num_q_tokens(self) -> int:
        return int(sum(self.q_lens))

    @property
    def max_query_len(self) -> int:
        return int(max(self.q_lens)) if self.q_lens else 0

    def query_start_loc(self) -> np.ndarray:
        qsl = np.zeros(len(self.q_lens) + 1, dtype=np.int32)
        qsl[1:] = np.cumsum(np.asarray(self.q_lens, dtype=np.int64))
        return qsl


class _Draw:
    """Independent seeded streams: lengths, values and the pool permutation."""

    def __init__(self, seed: int):
        ss = np.random.SeedSequence(seed)
        a, b, c = ss.spawn(3)
        self.lens = np.random.default_rng(a)
        self.vals = np.random.default_rng(b)
        self.perm = np.random.default_rng(c)

    def rows(self, n: int, heads: int, dim: int, dtype: str) -> np.ndarray:
        x = self.vals.standard_normal((n, heads, dim), dtype=np.float32)
        return f32_to_bf16_bits(x) if dtype == BF16 else x

    def pool_order(self, num_blocks: int, shuffled: bool = True) -> np.ndarray:
        if not shuffled:
            return np.arange(num_blocks, dtype=np.int32)
        return self.perm.permutation(num_blocks).astype(np.int32)


def _decode_batch(name, geo, ctx_lens, draw, notes=None, order=None) -> Workload:
    """Sequences of L tokens: L-1 stored up front, then 1 new token, then decode."""
    order = draw.pool_order(geo.num_blocks) if order is None else order
    ops = []
    for s, length in enumerate(ctx_lens):
        ops.append(Op("add", s, length - 1, k=draw.rows(length - 1, geo.num_kv_heads, geo.head_dim, geo.dtype),
                      v=draw.rows(length - 1, geo.num_kv_heads, geo.head_dim, geo.dtype)))
    for s in range(len(ctx_lens)):
        ops.append(Op("append", s, 1, k=draw.rows(1, geo.num_kv_heads, geo.head_dim, geo.dtype),
                      v=draw.rows(1, geo.num_kv_heads, geo.head_dim, geo.dtype)))
    q = draw.rows(len(ctx_lens), geo.num_q_heads, geo.head_dim, geo.dtype)
    return Workload(name, geo, order, ops, list(range(len(ctx_lens))), [1] * len(ctx_lens), q,
                    1.0 / math.sqrt(geo.head_dim), step_ops=len(ctx_lens),
                    notes=dict(notes or {}, context_lens=[int(x) for x in ctx_lens]))


# --------------------------------------------------------------------------
# the five configurations
# --------------------------------------------------------------------------

def tiny(seed: int = 0) -> Workload:
    """4 sequences, L = {5, 16, 17, 40}, bs 16, pool 16 blocks in a seeded random
    order, 4 q heads = 4 kv heads, head_dim 64, fp32, max 3 blocks per sequence."""
    geo = Geometry(16, 16, 4, 4, 64, FP32, 3)
    return _decode_batch("tiny_paged_decode_fp32", geo, [5, 16, 17, 40], _Draw(seed))


def llama7b_decode(seed: int = 0, num_blocks: int = 8192) -> Workload:
    """32 q = 32 kv heads, head_dim 128, bf16, pool 8192 blocks of 16 (1 GiB per
    cache), batch 32, L ~ U{128..2048}, blocks from a shuffled free list.
    ``num_blocks`` shrinks the pool (same lengths and values) for profiling
    captures that must hold little device memory."""
    draw = _Draw(seed)
    geo = Geometry(num_blocks, 16, 32, 32, 128, BF16, 128)
    lens = draw.lens.integers(128, 2048, size=32, endpoint=True)
    suffix = "" if num_blocks == 8192 else "_pool%d" % num_blocks
    return _decode_batch("llama7b_decode_b32_bf16" + suffix, geo, lens, draw)


def gqa_long_decode(seed: int = 0) -> Workload:
    """32 q / 8 kv heads, head_dim 128, bf16, bs 16, max 512 blocks per sequence,
    batch 16, L = clip(round(exp(ln 2048 + 0.5 N(0,1))), 256, 8192), pool 16384."""
    draw = _Draw(seed)
    geo = Geometry(16384, 16, 8, 32, 128, BF16, 512)
    z = draw.lens.standard_normal(16)
    lens = np.clip(np.round(np.exp(math.log(2048.0) + 0.5 * z)), 256, 8192).astype(np.int64)
    return _decode_batch("gqa_long_decode_b16_bf16", geo, lens, draw)


def prefix_cow_decode(seed: int = 0, prefix_len: int = 1992) -> Workload:
    """64 sequences: 48 share one ``prefix_len``-token prefix (1992 = 124 full
    blocks + 8 tokens, so the shared last block is partly filled and the first
    write of each sharer copies it), each with a private suffix of U{16..512}
    tokens; 16 unshared sequences with L ~ U{256..2048}. 32 q / 8 kv heads,
    head_dim 128, bf16, bs 16, pool 16384 shuffled blocks."""
    draw = _Draw(seed)
    geo = Geometry(16384, 16, 8, 32, 128, BF16, 160)
    hkv, d, dt = geo.num_kv_heads, geo.head_dim, geo.dtype
    suffix = draw.lens.integers(16, 512, size=48, endpoint=True)
    private = draw.lens.integers(256, 2048, size=16, endpoint=True)
    ops = [Op("add", 0, prefix_len, k=draw.rows(prefix_len, hkv, d, dt), v=draw.rows(prefix_len, hkv, d, dt))]
    for s in range(1, 48):
        ops.append(Op("fork", s, prefix_len, parent=0))
    for s in range(48):
        n = int(suffix[s]) - 1
        ops.append(Op("append", s, n, k=draw.rows(n, hkv, d, dt), v=draw.rows(n, hkv, d, dt)))
    for j in range(16):
        n = int(private[j]) - 1
        ops.append(Op("add", 48 + j, n, k=draw.rows(n, hkv, d, dt), v=draw.rows(n, hkv, d, dt)))
    for s in range(64):
        ops.append(Op("append", s, 1, k=draw.rows(1, hkv, d, dt), v=draw.rows(1, hkv, d, dt)))
    q = draw.rows(64, geo.num_q_heads, d, dt)
    lens = [prefix_len + int(x) for x in suffix] + [int(x) for x in private]
    return Workload("prefix_cow_decode_b64_bf16" + ("" if prefix_len == 1992 else "_p%d" % prefix_len),
                    geo, draw.pool_order(geo.num_blocks), ops, list(range(64)), [1] * 64, q,
                    1.0 / math.sqrt(d), step_ops=64,
                    notes=dict(prefix_len=prefix_len, context_lens=lens))


def mixed_prefill_decode(block_size: int = 16, seed: int = 0) -> Workload:
    """4 sequences each prefilling a 256-token chunk on top of c ~ U{0..1792}
    cached tokens, plus 28 decode sequences with L ~ U{256..4096}; prefill rows
    first in the packed batch (T = 4*256 + 28 = 1052). 32 q / 8 kv heads,
    head_dim 128, bf16. The pool holds 131072 tokens at every block size; the
    lengths and values are the same for block_size 8, 16 and 32."""
    draw = _Draw(seed)
    chunk = 256
    geo = Geometry(131072 // block_size, block_size, 8, 32, 128, BF16, -(-4096 // block_size))
    hkv, d, dt = geo.num_kv_heads, geo.head_dim, geo.dtype
    prior = draw.lens.integers(0, 1792, size=4, endpoint=True)
    dec = draw.lens.integers(256, 4096, size=28, endpoint=True)
    ops = []
    for s in range(4):
        c = int(prior[s])
        ops.append(Op("add", s, c, k=draw.rows(c, hkv, d, dt), v=draw.rows(c, hkv, d, dt)))
    for j in range(28):
        n = int(dec[j]) - 1
        ops.append(Op("add", 4 + j, n, k=draw.rows(n, hkv, d, dt), v=draw.rows(n, hkv, d, dt)))
    for s in range(4):
        ops.append(Op("append", s, chunk, k=draw.rows(chunk, hkv, d, dt), v=draw.rows(chunk, hkv, d, dt)))
    for j in range(28):
        ops.append(Op("append", 4 + j, 1, k=draw.rows(1, hkv, d, dt), v=draw.rows(1, hkv, d, dt)))
    q_lens = [chunk] * 4 + [1] * 28
    q = draw.rows(sum(q_lens), geo.num_q_heads, d, dt)
    lens = [int(c) + chunk for c in prior] + [int(x) for x in dec]
    return Workload("mixed_prefill_decode_bs%d_bf16" % block_size, geo, draw.pool_order(geo.num_blocks),
                    ops, list(range(32)), q_lens, q, 1.0 / math.sqrt(d), step_ops=32,
                    notes=dict(prior_context=[int(c) for c in prior], context_lens=lens))


def random_case(seed: int, *, num_seqs: int, q_lens, ctx_extra, num_kv_heads: int, group: int,
                head_dim: int, block_size: int, dtype: str, num_blocks: int | None = None,
                max_blocks_per_seq: int | None = None, shuffled: bool = True) -> Workload:
    """Small mixed batch for parity sweeps.

    Sequence s has ``ctx_extra[s]`` cached tokens plus ``q_lens[s]`` new tokens
    that are stored and then queried (so L = ctx_extra + q_len).
    """
    draw = _Draw(seed)
    lens = [int(c) + int(q) for c, q in zip(ctx_extra, q_lens)]
    need = sum(-(-x // block_size) for x in lens)
    nb = num_blocks if num_blocks is not None else need + 8
    mb = max_blocks_per_seq if max_blocks_per_seq is not None else max(1, max(-(-x // block_size) for x in lens))
    geo = Geometry(nb, block_size, num_kv_heads, num_kv_heads * group, head_dim, dtype, mb)
    ops = []
    for s in range(num_seqs):
        c = int(ctx_extra[s])
        ops.append(Op("add", s, c, k=draw.rows(c, num_kv_heads, head_dim, dtype),
                      v=draw.rows(c, num_kv_heads, head_dim, dtype)))
    for s in range(num_seqs):
        n = int(q_lens[s])
        ops.append(Op("append", s, n, k=draw.rows(n, num_kv_heads, head_dim, dtype),
                      v=draw.rows(n, num_kv_heads, head_dim, dtype)))
    q = draw.rows(int(sum(q_lens)), num_kv_heads * group, head_dim, dtype)
    return Workload("random_%d" % seed, geo, draw.pool_order(nb, shuffled), ops, list(range(num_seqs)),
                    [int(x) for x in q_lens], q, 1.0 / math.sqrt(head_dim), step_ops=num_seqs,
                    notes=dict(context_lens=lens))


def shared_prefix_case(seed: int, *, groups, singles, num_kv_heads: int, group: int, head_dim: int,
                       block_size: int, dtype: str, max_blocks_per_seq: int | None = None) -> Workload:
    """Decode batch with shared prefixes, for cascade parity.

    ``groups`` is a list of ``(prefix_len, [L_1, L_2, ...])``: the first member
    holds the prefix, the others fork it whole, and member i grows to L_i
    tokens (L_i > prefix_len; the last token is the step's decode row).
    ``singles`` are lengths of sequences that share nothing; they are placed
    between the groups (batch order: single, group 0, single, group 1, ...).
    """
    draw = _Draw(seed)
    hkv, d = num_kv_heads, head_dim
    order, lens, ops = [], [], []
    sid = 0
    singles = list(singles)
    for gi, (plen, member_lens) in enumerate(groups):
        if singles:
            L = int(singles.pop(0))
            ops.append(Op("add", sid, L - 1, k=draw.rows(L - 1, hkv, d, dtype), v=draw.rows(L - 1, hkv, d, dtype)))
            order.append(sid)
            lens.append(L)
            sid += 1
        lead = sid
        ops.append(Op("add", lead, plen, k=draw.rows(plen, hkv, d, dtype), v=draw.rows(plen, hkv, d, dtype)))
        for m, L in enumerate(member_lens):
            if m:
                ops.append(Op("fork", sid, plen, parent=lead))
            n = int(L) - plen - 1
            ops.append(Op("append", sid, n, k=draw.rows(n, hkv, d, dtype), v=draw.rows(n, hkv, d, dtype)))
            order.append(sid)
            lens.append(int(L))
            sid += 1
    for L in singles:
        ops.append(Op("add", sid, L - 1, k=draw.rows(L - 1, hkv, d, dtype), v=draw.rows(L - 1, hkv, d, dtype)))
        order.append(sid)
        lens.append(int(L))
        sid += 1
    for s in order:
        ops.append(Op("append", s, 1, k=draw.rows(1, hkv, d, dtype), v=draw.rows(1, hkv, d, dtype)))
    nb = sum(-(-L // block_size) for L in lens) + 8 * len(lens) + 8
    mb = max_blocks_per_seq or max(-(-L // block_size) for L in lens)
    geo = Geometry(nb, block_size, hkv, hkv * group, d, dtype, mb)
    q = draw.rows(len(order), hkv * group, d, dtype)
    return Workload("shared_prefix_%d" % seed, geo, draw.pool_order(nb), ops, order, [1] * len(order), q,
                    1.0 / math.sqrt(d), step_ops=len(order), notes=dict(context_lens=lens))


CONFIGS = {
    "tiny": tiny,
    "llama7b": llama7b_decode,
    "llama7b_pool2560": lambda seed=0: llama7b_decode(seed, 2560),
    "gqa_long": gqa_long_decode,
    "prefix_cow": prefix_cow_decode,
    "mixed_bs8": lambda seed=0: mixed_prefill_decode(8, seed),
    "mixed_bs16": lambda seed=0: mixed_prefill_decode(16, seed),
    "mixed_bs32": lambda seed=0: mixed_prefill_decode(32, seed),
}


# --------------------------------------------------------------------------
# initial cache contents
# --------------------------------------------------------------------------

#: Bit pattern every cache element holds before the first store: a quiet NaN.
#: Unwritten slots (the unfilled tail of a sequence's last block, blocks no
#: sequence owns) must keep it, and attention must never let it leak into a
#: result, since a real cache holds arbitrary stale bits there.
SENTINEL_BF16 = np.uint16(0x7FC1)
SENTINEL_FP32 = np.uint32(0x7FC00001)


def sentinel_cache(geo: Geometry) -> np.ndarray:
    """Host array ``[NB, bs, Hkv, D]`` filled with the sentinel pattern."""
    shape = (geo.num_blocks, geo.block_size, geo.num_kv_heads, geo.head_dim)
    if geo.dtype == BF16:
        return np.full(shape, SENTINEL_BF16, dtype=np.uint16)
    return np.full(shape, SENTINEL_FP32, dtype=np.uint32).view(np.float32)
