"""Pins for the oracle block manager (CPU only).

Pinned to the pages' worked numbers (tests/golden/pages_worked_examples.json),
to the invariants the pages state (a block is free exactly when no sequence
holds it; freeing at refcount 0 returns the block; a shared page is copied only
when written) and to brute-force enumeration on random operation sequences.
"""

import numpy as np
import pytest

import oracle
from oracle import BlockManager, OutOfBlocks
from paged_kv_cache_heads_b200 import workloads as W


def check_invariants(bm: BlockManager):
    """Free list and held blocks partition the pool; refcounts equal holder counts."""
    free = list(bm.free)
    assert len(set(free)) == len(free), "duplicate in free list"
    holders = np.zeros(bm.num_blocks, dtype=np.int64)
    for sid, row in bm.tables.items():
        for b in row:
            holders[b] += 1
        assert len(row) == -(-bm.lens[sid] // bm.block_size)
    assert list(holders) == list(bm.ref)
    held = {b for b in range(bm.num_blocks) if bm.ref[b] > 0}
    assert held.isdisjoint(free)
    assert len(held) + len(free) == bm.num_blocks


def test_short_generation_holds_only_its_pages(golden):
    ex = golden["short_generation"]
    bm = BlockManager(256, ex["block_size"])
    bm.add_seq(1, ex["generated_tokens"])
    assert len(bm.blocks_of(1)) == 4                       # ceil(50 / 16)
    assert len(bm.blocks_of(1)) * ex["block_size"] < ex["preallocated_tokens"]
    assert bm.num_free() == 256 - 4
    check_invariants(bm)


def test_128k_context_fills_8192_blocks_exactly(golden):
    ex = golden["blocks_for_128k"]
    bm = BlockManager(ex["stated_blocks"], ex["block_size"])
    bm.add_seq(0, ex["context_tokens"])
    assert bm.num_free() == 0 and len(bm.blocks_of(0)) == ex["stated_blocks"]
    with pytest.raises(OutOfBlocks):
        bm.append_tokens(0, 1)
    assert bm.seq_len(0) == ex["context_tokens"]          # unchanged by the failed append
    check_invariants(bm)


def test_max_blocks_per_seq_caps_context(golden):
    cfg = golden["default_config"]
    bm = BlockManager(cfg["max_blocks_per_seq"] + 1, cfg["block_size"])
    bm.add_seq(0, cfg["max_blocks_per_seq"] * cfg["block_size"])
    table, lens = bm.block_table([0], cfg["max_blocks_per_seq"])
    assert lens[0] == 8192 and (table >= 0).all()
    bm.append_tokens(0, 1)
    with pytest.raises(ValueError):
        bm.block_table([0], cfg["max_blocks_per_seq"])


def test_three_requests_share_prompt(golden):
    ex = golden["three_requests"]
    bs = 16
    P, Q = ex["reading_system_prompt_tokens"], ex["reading_question_tokens"]
    bm = BlockManager(512, bs)
    bm.add_seq(100, P)                                     # the cached system prompt
    bm.fork(100, 1, P)                                     # A
    bm.fork(100, 2, P)                                     # B
    bm.free_seq(100)
    bm.append_tokens(1, Q + ex["A"]["generated"])
    bm.append_tokens(2, Q + ex["B"]["generated"])
    bm.add_seq(3, Q + ex["C"]["generated"])               # C: no system prompt
    prompt_blocks = bm.blocks_of(1)[: P // bs]
    assert prompt_blocks == bm.blocks_of(2)[: P // bs]
    assert all(bm.refcount(b) == 2 for b in prompt_blocks)
    assert set(bm.blocks_of(3)).isdisjoint(bm.blocks_of(1) + bm.blocks_of(2))
    held_tokens = (512 - bm.num_free()) * bs
    assert held_tokens < ex["stated_max_fraction"] * 3 * ex["preallocated_tokens_each"]
    bm.free_seq(2)                                         # B finishes first
    assert all(bm.refcount(b) == 1 for b in prompt_blocks)
    assert not set(prompt_blocks) & set(bm.free)
    check_invariants(bm)


def test_free_at_refcount_zero_returns_blocks_in_order():
    bm = BlockManager(10, 4, initial_free_order=[9, 8, 7, 6, 5, 4, 3, 2, 1, 0])
    bm.add_seq(0, 10)                                      # blocks 9, 8, 7
    bm.fork(0, 1, 6)                                       # shares 9, 8
    bm.free_seq(0)
    assert list(bm.free)[-1:] == [7]                       # only 7 reached refcount 0
    assert bm.refcount(9) == 1 and bm.refcount(8) == 1
    bm.free_seq(1)
    assert list(bm.free)[-3:] == [7, 9, 8]
    check_invariants(bm)


def test_copy_on_write_only_for_shared_partial_block():
    bm = BlockManager(20, 4, initial_free_order=list(range(20)))
    bm.add_seq(0, 6)                                       # blocks 0, 1 (block 1 half full)
    bm.fork(0, 1)
    bm.fork(0, 2)
    assert bm.refcount(1) == 3
    slots, pairs = bm.append_tokens(1, 1)                 # shared partial block -> copy
    assert pairs == [(1, 2)] and bm.blocks_of(1) == [0, 2] and slots == [2 * 4 + 2]
    assert bm.refcount(1) == 2 and bm.refcount(2) == 1
    slots, pairs = bm.append_tokens(1, 1)                 # now private: no copy
    assert pairs == [] and slots == [2 * 4 + 3]
    _, pairs = bm.append_tokens(2, 3)
    assert pairs == [(1, 3)]
    _, pairs = bm.append_tokens(0, 1)                     # last holder writes in place
    assert pairs == [] and bm.blocks_of(0) == [0, 1]
    check_invariants(bm)


def test_block_aligned_share_needs_no_copy():
    bm = BlockManager(10, 4)
    bm.add_seq(0, 8)
    bm.fork(0, 1)
    _, pairs = bm.append_tokens(1, 5)
    assert pairs == [] and bm.blocks_of(1)[:2] == bm.blocks_of(0)
    check_invariants(bm)


def test_failed_operations_change_nothing():
    bm = BlockManager(5, 4)
    bm.add_seq(0, 7)
    bm.fork(0, 1)
    before = (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.lens))
    with pytest.raises(OutOfBlocks):
        bm.append_tokens(1, 14)                            # needs a copy + 3 new blocks, 3 free
    with pytest.raises(OutOfBlocks):
        bm.add_seq(2, 13)
    with pytest.raises(ValueError):
        bm.add_seq(0, 1)
    with pytest.raises(ValueError):
        bm.fork(0, 1)
    with pytest.raises(ValueError):
        bm.free_seq(7)
    after = (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.lens))
    assert before == after


def test_prefix_config_copy_count():
    """48 sharers of a 1992-token prefix: 47 copies, the last sharer writes in place;
    a 2000-token (block-aligned) prefix needs none."""
    for P, expect in ((1992, 47), (2000, 0)):
        wl = W.prefix_cow_decode(prefix_len=P)
        bm = BlockManager(wl.geometry.num_blocks, 16, wl.initial_free_order)
        n_pairs = 0
        for op in wl.ops:
            if op.kind == "add":
                bm.add_seq(op.seq, op.n)
            elif op.kind == "fork":
                bm.fork(op.parent, op.seq, op.n)
            elif op.kind == "append":
                n_pairs += len(bm.append_tokens(op.seq, op.n)[1])
        assert n_pairs == expect
        check_invariants(bm)


def test_slots_enumerate_sequence_blocks():
    """Brute force: the slots of a sequence are exactly the slots of its blocks, in order."""
    rng = np.random.default_rng(9)
    bm = BlockManager(64, 8, initial_free_order=rng.permutation(64))
    slots = bm.add_seq(0, 29)
    expect = [b * 8 + o for b in bm.blocks_of(0) for o in range(8)][:29]
    assert slots == expect
    assert bm.slot_mapping(0, 5, 10) == expect[5:15]


@pytest.mark.parametrize("seed", range(6))
def test_random_operation_sequences_keep_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    bs = int(rng.choice([4, 8, 16]))
    nb = int(rng.integers(8, 80))
    bm = BlockManager(nb, bs, initial_free_order=rng.permutation(nb))
    live, next_id = [], 0
    for _ in range(300):
        r = rng.random()
        try:
            if r < 0.3 or not live:
                bm.add_seq(next_id, int(rng.integers(0, 3 * bs)))
                live.append(next_id)
                next_id += 1
            elif r < 0.45:
                p = int(rng.choice(live))
                bm.fork(p, next_id, int(rng.integers(0, bm.seq_len(p) + 1)))
                live.append(next_id)
                next_id += 1
            elif r < 0.85:
                s = int(rng.choice(live))
                before = bm.blocks_of(s)
                L0 = bm.seq_len(s)
                n = int(rng.integers(0, 2 * bs))
                slots, pairs = bm.append_tokens(s, n)
                after = bm.blocks_of(s)
                assert len(slots) == n and len(pairs) <= 1
                for p_, sl in zip(range(L0, L0 + n), slots):
                    assert sl == after[p_ // bs] * bs + p_ % bs
                for old, new in pairs:
                    assert old == before[-1] and after[len(before) - 1] == new
            else:
                s = int(rng.choice(live))
                bm.free_seq(s)
                live.remove(s)
        except OutOfBlocks:
            pass
        check_invariants(bm)
    for s in list(live):
        bm.free_seq(s)
    assert bm.num_free() == nb and sorted(bm.free) == list(range(nb))


# --------------------------------------------------------------------------
# monitoring figures ([A] §"监控与调优要点")
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n,bs", [(0, 16), (1, 16), (16, 16), (17, 16), (50, 16), (2047, 32), (5, 8)])
def test_stats_single_sequence_closed_form(n, bs):
    bm = BlockManager(300, bs)
    bm.add_seq(0, n)
    st = bm.stats()
    blocks = -(-n // bs)
    assert st["held_blocks"] == st["logical_blocks"] == blocks
    assert st["used_slots"] == st["tokens"] == n
    assert st["block_utilisation"] == blocks / 300
    want_frag = (blocks * bs - n) / (blocks * bs) if blocks else 0.0
    assert st["internal_fragmentation"] == pytest.approx(want_frag, abs=1e-15)
    assert st["sharing_saving"] == 0.0 and st["table_bytes"] == 4 * blocks


@pytest.mark.parametrize("children", [1, 3, 7])
def test_stats_full_fork_shares_every_slot(children):
    bm = BlockManager(64, 16)
    bm.add_seq(0, 40)                                      # 3 blocks, 8 slots empty
    for c in range(children):
        bm.fork(0, c + 1)
    st = bm.stats()
    assert st["held_blocks"] == 3 and st["logical_blocks"] == 3 * (children + 1)
    assert st["tokens"] == 40 * (children + 1)
    assert st["used_slots"] == 40                          # a shared slot counts once
    assert st["internal_fragmentation"] == pytest.approx(8 / 48, abs=1e-15)
    assert st["sharing_saving"] == pytest.approx(1 - 1 / (children + 1), abs=1e-15)


def test_stats_after_copy_on_write_and_short_fork():
    bm = BlockManager(16, 4)
    bm.add_seq(0, 10)                                      # blocks b0 b1 b2 (2 in b2)
    bm.fork(0, 1, 6)                                       # shares b0, b1 (2 of b1's 4 tokens)
    st = bm.stats()
    assert st["held_blocks"] == 3 and st["used_slots"] == 10 and st["logical_blocks"] == 5
    bm.append_tokens(1, 1)                                 # CoW of b1: a private copy holding 3 tokens
    st = bm.stats()
    assert st["held_blocks"] == 4 and st["used_slots"] == 10 + 3
    assert st["internal_fragmentation"] == pytest.approx(1 - 13 / 16, abs=1e-15)
    bm.free_seq(0)                                         # b1 and b2 go back; b0 stays with seq 1
    st = bm.stats()
    assert st["held_blocks"] == 2 and st["used_slots"] == 7 and st["free_blocks"] == 14


def test_stats_table_of_a_128k_context(golden):
    """8192 table entries of one int32 for the page's 128K context at 16 tokens a block."""
    ex = golden["blocks_for_128k"]
    kv = golden["kv_per_request"]
    per_block = oracle.kv_bytes_per_token(kv["num_layers"], kv["hidden_size"] // 128, 128,
                                          kv["elem_bytes_fp16"]) * ex["block_size"]
    bm = BlockManager(ex["stated_blocks"], ex["block_size"])
    bm.add_seq(0, ex["context_tokens"])
    st = bm.stats(per_block)
    assert st["table_bytes"] == 4 * ex["stated_blocks"]
    assert st["block_utilisation"] == 1.0 and st["internal_fragmentation"] == 0.0
    # the page's guidance: the mapping table stays well under 1% of the KV cache
    assert st["table_overhead"] == pytest.approx(4 / per_block, rel=1e-12) and st["table_overhead"] < 0.01


def test_stats_paged_vs_preallocated_fragmentation_on_decode_batch():
    """[C] §"二、KV Cache管理：从浪费到极致复用" table: internal fragmentation
    under 5% with pages against up to 60% when each request reserves the
    maximum length; recomputed on the 32-sequence decode batch (lengths
    128..2048, 16 tokens a block, 2048-token reservation)."""
    wl = W.llama7b_decode()
    geo = wl.geometry
    bm = BlockManager(geo.num_blocks, geo.block_size, wl.initial_free_order)
    for op in wl.ops:
        if op.kind == "add":
            bm.add_seq(op.seq, op.n)
        elif op.kind == "append":
            bm.append_tokens(op.seq, op.n)
    st = bm.stats()
    assert st["internal_fragmentation"] < 0.05
    pre = oracle.preallocation_fragmentation([bm.seq_len(s) for s in wl.batch_seqs], 2048)
    assert 0.05 < pre <= 0.60
    assert pre == pytest.approx(1 - st["tokens"] / (len(wl.batch_seqs) * 2048), abs=1e-15)


def test_preallocation_fragmentation_pinned_to_the_pages_example(golden):
    """[C] §"二、KV Cache管理：从浪费到极致复用": a request that generates 50 tokens
    under a scheme that reserves 2048 slots per request leaves 1998 of its
    2048 slots unused (worked by hand: 2048 - 50 = 1998)."""
    ex = golden["short_generation"]
    n, reserved = ex["generated_tokens"], ex["preallocated_tokens"]
    assert (n, reserved) == (50, 2048)
    assert oracle.preallocation_fragmentation([n], reserved) == 1998 / 2048
    # a second request that fills its whole reservation wastes nothing:
    # 1998 unused slots out of 2 x 2048 reserved
    assert oracle.preallocation_fragmentation([n, reserved], reserved) == 1998 / 4096
    # closed forms: every request full -> 0; no tokens at all -> 1
    assert oracle.preallocation_fragmentation([reserved] * 3, reserved) == 0.0
    assert oracle.preallocation_fragmentation([0, 0], reserved) == 1.0


def test_preallocation_fragmentation_planted_slip_fails():
    """Dividing by the batch's longest request instead of the reservation (a
    plausible slip) gives 1/4 here, not 1 - 150/4096."""
    lens = [50, 100]
    slip = 1.0 - sum(lens) / (len(lens) * max(lens))
    assert slip == 0.25
    assert oracle.preallocation_fragmentation(lens, 2048) == 1.0 - 150 / 4096 != slip


def test_stats_count_planted_double_counting():
    """A plausible slip, counting a shared slot once per holder, breaks the fork pin."""
    bm = BlockManager(8, 4)
    bm.add_seq(0, 6)
    bm.fork(0, 1)
    per_holder = sum(bm.seq_len(s) for s in bm.tables)
    assert per_holder == 12 and bm.stats()["used_slots"] == 6


# --------------------------------------------------------------------------
# compaction ([A] §"连续批处理与内存管理的协同": remap blocks, weigh the moves)
# --------------------------------------------------------------------------

def _scattered_pool(seed, nb=64, bs=4):
    rng = np.random.default_rng(seed)
    bm = BlockManager(nb, bs, rng.permutation(nb))
    for s in range(12):
        bm.add_seq(s, int(rng.integers(0, 5 * bs)))
    bm.fork(3, 100)
    bm.fork(5, 101, max(0, bm.seq_len(5) - 3))
    bm.append_tokens(101, 2)
    for s in (0, 4, 7, 9):
        bm.free_seq(s)
    return bm


@pytest.mark.parametrize("seed", range(6))
def test_compaction_makes_held_blocks_dense_and_keeps_every_token(seed):
    bm = _scattered_pool(seed)
    bs = bm.block_size
    # give every slot a value that names (block, row), then move the data as the pairs say
    cache = np.arange(bm.num_blocks * bs, dtype=np.int64).reshape(bm.num_blocks, bs)
    before = {s: [cache[b, p % bs] for p in range(bm.seq_len(s)) for b in [bm.blocks_of(s)[p // bs]]]
              for s in bm.tables}
    refs_before = sorted(bm.ref[b] for b in range(bm.num_blocks) if bm.ref[b] > 0)
    held = sum(1 for b in range(bm.num_blocks) if bm.ref[b] > 0)
    pairs = bm.compact()
    for src, dst in pairs:
        assert src >= held > dst                        # moves only from above the dense range into it
        cache[dst] = cache[src]
    assert len({d for _, d in pairs}) == len(pairs) == len({s for s, _ in pairs})
    assert {b for b in range(bm.num_blocks) if bm.ref[b] > 0} == set(range(held))
    assert list(bm.free) == list(range(held, bm.num_blocks))
    assert sorted(bm.ref[b] for b in range(held)) == refs_before
    after = {s: [cache[b, p % bs] for p in range(bm.seq_len(s)) for b in [bm.blocks_of(s)[p // bs]]]
             for s in bm.tables}
    assert after == before
    check_invariants(bm)
    assert bm.compact() == []                           # already dense: nothing moves


def test_compaction_order_is_ascending_movers_to_ascending_holes():
    bm = BlockManager(8, 2, [7, 5, 3, 0, 1, 2, 4, 6])
    bm.add_seq(0, 4)                                    # blocks 7, 5
    bm.add_seq(1, 2)                                    # block 3
    # H = 3 held blocks, all at ids >= 3: 3 -> 0, 5 -> 1, 7 -> 2
    assert bm.compact() == [(3, 0), (5, 1), (7, 2)]
    assert bm.blocks_of(0) == [2, 1] and bm.blocks_of(1) == [0]
    assert list(bm.free) == [3, 4, 5, 6, 7]


# --------------------------------------------------------------------------
# cascade groups ([C] §"二、KV Cache管理：从浪费到极致复用": shared prefix pages)
# --------------------------------------------------------------------------

def _replay_bm(wl):
    geo = wl.geometry
    bm = BlockManager(geo.num_blocks, geo.block_size, wl.initial_free_order)
    for op in wl.ops:
        if op.kind == "add":
            bm.add_seq(op.seq, op.n)
        elif op.kind == "fork":
            bm.fork(op.parent, op.seq, op.n)
        elif op.kind == "append":
            bm.append_tokens(op.seq, op.n)
    return bm


def test_cascade_groups_hand_case():
    # group 0: 64-token prefix = 4 full blocks of 16, members of 70, 100, 65 tokens;
    # group 1: 37-token prefix = 2 full blocks (its third block is copied on write);
    # unshared sequences of 5, 90, 17 tokens sit before each group and at the end
    wl = W.shared_prefix_case(3, groups=[(64, [70, 100, 65]), (37, [40, 41])], singles=[5, 90, 17],
                              num_kv_heads=2, group=4, head_dim=128, block_size=16, dtype=W.BF16)
    bm = _replay_bm(wl)
    shared, groups = bm.cascade_groups(wl.batch_seqs)
    assert groups == [(1, 3), (5, 2)]
    assert shared == [0, 4, 4, 4, 0, 2, 2, 0]
    # a stricter threshold keeps only the 4-block group
    shared, groups = bm.cascade_groups(wl.batch_seqs, min_shared_blocks=3)
    assert groups == [(1, 3)] and shared == [0, 4, 4, 4, 0, 0, 0, 0]


def test_cascade_groups_prefix_config():
    """The shared-prompt configuration: 48 sequences share 124 full blocks
    (1992 tokens = 124 * 16 + 8; the partly filled 125th block is copied on
    each sharer's first write)."""
    wl = W.prefix_cow_decode()
    bm = _replay_bm(wl)
    shared, groups = bm.cascade_groups(wl.batch_seqs)
    assert groups == [(0, 48)]
    assert shared == [124] * 48 + [0] * 16
    lead = bm.blocks_of(0)[:124]
    assert all(bm.blocks_of(s)[:124] == lead for s in range(48))
