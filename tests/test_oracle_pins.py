"""Pins for the oracle's store, copy, indexing and attention (CPU only).

Each pin ties the oracle to something other than itself: values the pages
print, closed forms, a library routine on an equivalent contiguous problem,
brute force on tiny inputs, or an invariant the method guarantees. The
mutation tests at the end plant plausible mistakes in copies of the oracle and
check that at least one pin catches each.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import paged_kv as OA
from paged_kv_cache_heads_b200 import workloads as W


# --------------------------------------------------------------------------
# helpers building small paged problems directly (no block manager)
# --------------------------------------------------------------------------

def _paged_problem(rng, lens, q_lens, hkv, g, d, bs, extra_blocks=3, dtype=np.float64):
    """Random contiguous K/V per sequence, scattered into a shuffled pool."""
    nblk = [-(-L // bs) for L in lens]
    nb = sum(nblk) + extra_blocks
    perm = rng.permutation(nb)
    kc = rng.standard_normal((nb, bs, hkv, d)).astype(dtype)
    vc = rng.standard_normal((nb, bs, hkv, d)).astype(dtype)
    mb = max(nblk)
    tables = np.full((len(lens), mb), -1, dtype=np.int64)
    kcont, vcont = [], []
    at = 0
    for s, L in enumerate(lens):
        blocks = perm[at:at + nblk[s]]
        at += nblk[s]
        tables[s, :nblk[s]] = blocks
        kk = rng.standard_normal((L, hkv, d))
        vv = rng.standard_normal((L, hkv, d))
        for i in range(L):
            kc[blocks[i // bs], i % bs] = kk[i]
            vc[blocks[i // bs], i % bs] = vv[i]
        kcont.append(kk)
        vcont.append(vv)
    qsl = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int64)
    q = rng.standard_normal((int(qsl[-1]), hkv * g, d))
    return q, kc, vc, tables, np.asarray(lens), qsl, kcont, vcont


def _sdpa_reference(q, kcont, vcont, lens, qsl, scale, g):
    """torch SDPA (float64, CPU) on the contiguous sequences with an explicit mask."""
    out = np.zeros_like(q)
    for s, L in enumerate(lens):
        r0, r1 = int(qsl[s]), int(qsl[s + 1])
        ql = r1 - r0
        if ql == 0:
            continue
        qq = torch.from_numpy(q[r0:r1]).permute(1, 0, 2)                      # [Hq, ql, D]
        kk = torch.from_numpy(kcont[s]).permute(1, 0, 2).repeat_interleave(g, 0)  # [Hq, L, D]
        vv = torch.from_numpy(vcont[s]).permute(1, 0, 2).repeat_interleave(g, 0)
        pos = L - ql + torch.arange(ql)
        mask = torch.arange(L)[None, :] <= pos[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale)
        out[r0:r1] = o.permute(1, 0, 2).numpy()
    return out


CASES = [
    # lens, q_lens, hkv, g, d, bs
    ([5, 16, 17, 40], [1, 1, 1, 1], 2, 1, 8, 16),
    ([3, 33, 20], [3, 7, 1], 2, 2, 16, 8),
    ([64, 9, 50, 31], [1, 9, 16, 2], 1, 4, 8, 32),
]


def _check_pins(attn, seed=0):
    """Return a list of failed pin names for attention implementation ``attn``."""
    failed = []
    rng = np.random.default_rng(seed)
    for ci, (lens, ql, hkv, g, d, bs) in enumerate(CASES):
        q, kc, vc, tb, L, qsl, kcont, vcont = _paged_problem(rng, lens, ql, hkv, g, d, bs)
        scale = 1.0 / math.sqrt(d)
        got = attn(q, kc, vc, tb, L, qsl, scale)
        # P2: equals contiguous attention computed by a library routine
        ref = _sdpa_reference(q, kcont, vcont, lens, qsl, scale, g)
        if not np.allclose(got, ref, rtol=0, atol=1e-12):
            failed.append("P2-sdpa-%d" % ci)
        # P1: invariant to any relabelling of physical blocks
        nb = kc.shape[0]
        pi = rng.permutation(nb)
        kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
        kc2[pi], vc2[pi] = kc, vc
        tb2 = np.where(tb >= 0, pi[np.maximum(tb, 0)], -1)
        if not np.array_equal(attn(q, kc2, vc2, tb2, L, qsl, scale), got):
            failed.append("P1-permutation-%d" % ci)
    # P3: identical keys give uniform weights, so each row is the mean of its visible V
    lens, ql, hkv, g, d, bs = [20, 7], [4, 1], 2, 2, 8, 8
    q, kc, vc, tb, L, qsl, kcont, vcont = _paged_problem(rng, lens, ql, hkv, g, d, bs)
    kc[:] = rng.standard_normal(d)
    got = attn(q, kc, vc, tb, L, qsl, 0.37)
    for s, Ls in enumerate(lens):
        for j in range(ql[s]):
            p = Ls - ql[s] + j
            vals = np.stack([vc[tb[s][i // bs], i % bs] for i in range(p + 1)])     # [p+1, Hkv, D]
            mean = vals.mean(axis=0).repeat(g, axis=0)                              # [Hq, D]
            if not np.allclose(got[qsl[s] + j], mean, rtol=0, atol=1e-12):
                failed.append("P3-identical-keys")
    # P5a: a single key gives o = v
    q, kc, vc, tb, L, qsl, kcont, vcont = _paged_problem(rng, [1], [1], 2, 2, 8, 16)
    got = attn(q, kc, vc, tb, L, qsl, 0.125)
    if not np.allclose(got[0], vc[tb[0][0], 0].repeat(2, axis=0), rtol=0, atol=1e-15):
        failed.append("P5-single-key")
    # P5b: scale 0 gives the mean of V
    q, kc, vc, tb, L, qsl, kcont, vcont = _paged_problem(rng, [19], [1], 1, 1, 8, 8)
    got = attn(q, kc, vc, tb, L, qsl, 0.0)
    if not np.allclose(got[0, 0], vcont[0][:, 0].mean(axis=0), rtol=0, atol=1e-12):
        failed.append("P5-scale0")
    # P5c: a decode row equals the last row of a prefill chunk over the same keys
    q, kc, vc, tb, L, qsl, kcont, vcont = _paged_problem(rng, [37], [5], 2, 2, 8, 16)
    full = attn(q, kc, vc, tb, L, qsl, 0.3)
    one = attn(q[4:5], kc, vc, tb, L, np.array([0, 1]), 0.3)
    if not np.allclose(full[4], one[0], rtol=0, atol=1e-13):
        failed.append("P5-decode-equals-last-prefill-row")
    return failed


def test_oracle_attention_passes_all_pins():
    assert _check_pins(oracle.paged_attention) == []


def test_bruteforce_matches_oracle_on_tiny_cases():
    rng = np.random.default_rng(3)
    for lens, ql, hkv, g, d, bs in CASES[:2]:
        q, kc, vc, tb, L, qsl, _, _ = _paged_problem(rng, lens, ql, hkv, g, d, bs)
        a = oracle.paged_attention(q, kc, vc, tb, L, qsl, 0.25)
        b = oracle.paged_attention_bruteforce(q, kc, vc, tb, L, qsl, 0.25)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_bruteforce_on_tiny_config_fp32():
    wl = W.tiny()
    from oracle import scenario
    kc, vc = W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry)
    run = scenario.run(wl, kc, vc)
    b = oracle.paged_attention_bruteforce(wl.q, run.k_cache, run.v_cache, run.block_tables,
                                          run.context_lens, run.query_start_loc, wl.scale)
    np.testing.assert_allclose(run.out, b, rtol=0, atol=1e-12)
    assert np.isfinite(run.out).all()


def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(5)
    q, kc, vc, tb, L, qsl, _, _ = _paged_problem(rng, [21, 8], [3, 1], 2, 4, 8, 8)
    gqa = oracle.paged_attention(q, kc, vc, tb, L, qsl, 0.2)
    mha = oracle.paged_attention(q, np.repeat(kc, 4, axis=2), np.repeat(vc, 4, axis=2), tb, L, qsl, 0.2)
    np.testing.assert_allclose(gqa, mha, rtol=0, atol=0)


def test_block_size_invariance_on_mixed_config():
    """The mixed config draws the same tokens at bs 8/16/32; fp64 results agree."""
    from oracle import scenario
    outs = []
    for bs in (8, 16, 32):
        wl = W.random_case(11, num_seqs=3, q_lens=[6, 1, 1], ctx_extra=[10, 40, 0], num_kv_heads=2,
                           group=2, head_dim=16, block_size=bs, dtype=W.FP32)
        run = scenario.run(wl, W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry))
        outs.append(run.out)
    np.testing.assert_allclose(outs[0], outs[1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(outs[0], outs[2], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# store / copy / indexing
# --------------------------------------------------------------------------

def test_store_matches_bruteforce_and_keeps_sentinels():
    rng = np.random.default_rng(1)
    geo = W.Geometry(6, 8, 2, 2, 8, W.BF16, 6)
    kc, vc = W.sentinel_cache(geo), W.sentinel_cache(geo)
    kc2, vc2 = kc.copy(), vc.copy()
    k = rng.integers(0, 2 ** 16, size=(10, 2, 8)).astype(np.uint16)
    v = rng.integers(0, 2 ** 16, size=(10, 2, 8)).astype(np.uint16)
    slots = rng.permutation(48)[:10].astype(np.int64)
    slots[[2, 7]] = -1
    oracle.store_kv(kc, vc, k, v, slots)
    oracle.store_kv_bruteforce(kc2, vc2, k, v, slots)
    assert np.array_equal(kc, kc2) and np.array_equal(vc, vc2)
    written = set(int(s) for s in slots if s >= 0)
    flat = kc.reshape(48, -1)
    for s in range(48):
        if s not in written:
            assert (flat[s] == W.SENTINEL_BF16).all()


def test_store_rejects_duplicate_slots():
    geo = W.Geometry(2, 4, 1, 1, 4, W.FP32, 2)
    kc, vc = W.sentinel_cache(geo), W.sentinel_cache(geo)
    k = np.ones((2, 1, 4), np.float32)
    with pytest.raises(ValueError):
        oracle.store_kv(kc, vc, k, k, np.array([3, 3]))


def test_copy_blocks_elementwise():
    rng = np.random.default_rng(2)
    kc = rng.standard_normal((8, 4, 2, 4)).astype(np.float32)
    vc = rng.standard_normal((8, 4, 2, 4)).astype(np.float32)
    k0, v0 = kc.copy(), vc.copy()
    pairs = [(1, 5), (3, 0), (1, 7)]
    oracle.copy_blocks(kc, vc, pairs)
    for b in range(8):
        src = {5: 1, 0: 3, 7: 1}.get(b, b)
        for o in range(4):
            for h in range(2):
                for e in range(4):
                    assert kc[b, o, h, e] == k0[src, o, h, e]
                    assert vc[b, o, h, e] == v0[src, o, h, e]
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, [(1, 2), (2, 3)])      # chained
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, [(1, 2), (3, 2)])      # repeated destination


def test_slot_of_round_trips_through_block_walk():
    """Write token ids through slot_of, read them back by walking the table."""
    rng = np.random.default_rng(4)
    for bs in (8, 16, 32):
        nb, L = 12, 5 * bs - 3
        table = rng.permutation(nb)[: -(-L // bs)]
        cache = np.full((nb, bs, 1, 1), -1, dtype=np.int64)
        for p in range(L):
            s = oracle.slot_of(table, p, bs)
            cache.reshape(nb * bs, 1)[s, 0] = p
        walked = OA._gather(cache, table, L)[:, 0, 0]
        assert list(walked) == list(range(L))


def test_kv_bytes_per_token_matches_pages_worked_example(golden):
    ex = golden["kv_per_request"]
    # hidden 4096 = heads x head_dim; the byte count does not depend on the split
    per_token = oracle.kv_bytes_per_token(ex["num_layers"], 32, ex["hidden_size"] // 32, ex["elem_bytes_fp16"])
    total = per_token * ex["seq_len"]
    assert abs(total - ex["approx_bytes"]) / ex["approx_bytes"] < ex["rel_tol"]
    assert oracle.kv_bytes_per_token(ex["num_layers"], 64, 64, 2) == per_token


# --------------------------------------------------------------------------
# planted mistakes: each mutant of the attention oracle must fail a pin
# --------------------------------------------------------------------------

def _mutant(kind):
    def attn(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale):
        q64 = OA.as_f64(q)
        t_total, hq, d = q64.shape
        hkv = k_cache.shape[2]
        g = hq // hkv
        out = np.zeros((t_total, hq, d))
        for s in range(len(context_lens)):
            L = int(context_lens[s])
            r0, r1 = int(query_start_loc[s]), int(query_start_loc[s + 1])
            ql = r1 - r0
            if ql == 0:
                continue
            off = 1 if kind == "causal_off_by_one" else 0
            pos = L - ql + np.arange(ql) - off
            vis = np.arange(L)[None, :] <= pos[:, None]
            if kind == "no_causal":
                vis = np.ones_like(vis)
            ka = OA.as_f64(OA._gather(k_cache, block_tables[s], L))
            va = OA.as_f64(OA._gather(v_cache, block_tables[s], L))
            if kind == "table_ignored":
                nblk = -(-L // k_cache.shape[1])
                ka = OA.as_f64(k_cache[:nblk].reshape(-1, hkv, d)[:L])
            for h in range(hq):
                kvh = (h % hkv) if kind == "head_map_mod" else h // g
                sc = 1.0 if kind == "no_scale" else scale
                lg = (q64[r0:r1, h] @ ka[:, kvh].T) * sc
                lg = np.where(vis, lg, -np.inf)
                lg = lg - lg.max(axis=1, keepdims=True)
                w = np.exp(lg)
                if kind != "no_normalise":
                    w = w / w.sum(axis=1, keepdims=True)
                vv = ka[:, kvh] if kind == "k_for_v" else va[:, kvh]
                out[r0:r1, h] = w @ vv
        return out
    return attn


@pytest.mark.parametrize("kind", ["causal_off_by_one", "no_causal", "table_ignored", "head_map_mod",
                                  "no_scale", "no_normalise", "k_for_v"])
def test_pins_catch_planted_mistake(kind):
    assert _check_pins(_mutant(kind)) != [], kind


def test_unmutated_copy_passes_pins():
    assert _check_pins(_mutant("none")) == []
