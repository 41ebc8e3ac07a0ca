"""GPU parity: libpa against the oracle on the same seeded workloads.

Store, copy and all block-table / slot indexing must match bit for bit;
attention must be within max |err| 2e-2 and mean |err| 2e-3 of the fp64
oracle for bf16 inputs (fp32 accumulation), and within 1e-4 for fp32 inputs.
The named configurations run at full size through the same calls the bench
times; the random sweep covers every supported dtype / head_dim / block size
and GQA grouping with ragged lengths and multi-split sequences.
"""

import os

import numpy as np
import pytest

import oracle
from oracle import scenario as oscen
from paged_kv_cache_heads_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {W.BF16: (2e-2, 2e-3), W.FP32: (1e-4, 1e-5)}


@pytest.fixture(scope="module")
def P():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_heads_b200 as P
    P.load_library()
    P.pa_read_device_flags(clear=True)
    return P


def _check_attention(got, ref, dtype, ctx=""):
    amax, amean = TOL[dtype]
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), "non-finite output " + ctx
    assert err.max() <= amax, "max err %.3g %s" % (err.max(), ctx)
    assert err.mean() <= amean, "mean err %.3g %s" % (err.mean(), ctx)
    return float(err.max()), float(err.mean())


def _run_both(P, wl, check_caches=True):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    kc, vc = W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry)
    o = oscen.run(wl, kc, vc)
    # indexing: identical slots, copy pairs, tables and lengths
    assert b.host["op_slots"] == [list(map(int, s)) for s in o.op_slots]
    assert [[tuple(p) for p in ps] for ps in b.host["op_pairs"]] == [[tuple(p) for p in ps] for ps in o.op_pairs]
    assert np.array_equal(b.host["block_tables"], o.block_tables)
    assert np.array_equal(b.host["context_lens"], o.context_lens)
    if check_caches:
        want_k = o.k_cache.view(np.uint16 if wl.geometry.dtype == W.BF16 else np.uint32)
        want_v = o.v_cache.view(np.uint16 if wl.geometry.dtype == W.BF16 else np.uint32)
        assert np.array_equal(gs.cache_bits(b.k_cache), want_k)
        assert np.array_equal(gs.cache_bits(b.v_cache), want_v)
    got = gs.out_as_f64(b.out, wl.geometry.dtype)
    flags = P.pa_read_device_flags(clear=True)
    assert flags == 0, hex(flags)
    return b, o, got


@pytest.mark.parametrize("name", ["tiny", "llama7b", "gqa_long", "prefix_cow", "prefix_cow_p2000"])
def test_config_parity(P, name):
    wl = W.prefix_cow_decode(prefix_len=2000) if name == "prefix_cow_p2000" else W.CONFIGS[name]()
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, wl.geometry.dtype, name)
    if name == "prefix_cow":
        assert sum(len(p) for p in o.op_pairs) == 47
    if name == "prefix_cow_p2000":
        assert sum(len(p) for p in o.op_pairs) == 0


def _random_decode(seed, dtype, d, bs, g, hkv=2, nseq=7):
    rng = np.random.default_rng(seed)
    lens = [1, bs, bs + 1, int(rng.integers(2, 3 * bs)), int(rng.integers(600, 1400)),
            int(rng.integers(1, 64)), int(rng.integers(2000, 2600))][:nseq]
    return W.random_case(seed, num_seqs=len(lens), q_lens=[1] * len(lens), ctx_extra=[x - 1 for x in lens],
                         num_kv_heads=hkv, group=g, head_dim=d, block_size=bs, dtype=dtype)


@pytest.mark.parametrize("dtype", [W.BF16, W.FP32])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("g", [1, 2, 3, 4, 8])
def test_random_decode_sweep(P, dtype, d, bs, g):
    wl = _random_decode(1000 + d + bs + 7 * g, dtype, d, bs, g)
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, dtype, "dtype=%s d=%d bs=%d g=%d" % (dtype, d, bs, g))


@pytest.mark.parametrize("dtype", [W.BF16, W.FP32])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_random_decode_multihead_sweep(P, dtype, d, bs):
    """No GQA and a multiple of 4 KV heads: each CTA streams 4 adjacent heads."""
    wl = _random_decode(3000 + d + bs, dtype, d, bs, 1, hkv=8)
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, dtype, "multihead dtype=%s d=%d bs=%d" % (dtype, d, bs))


@pytest.mark.parametrize("grid", ["1", "7", "64"])
def test_grid_partition_does_not_change_result(P, grid, monkeypatch):
    """Fewer decode CTAs move the partition boundaries (1 CTA: nothing is split)."""
    monkeypatch.setenv("PA_DECODE_GRID", grid)
    wl = _random_decode(77, W.BF16, 128, 16, 4)
    b, o, got = _run_both(P, wl, check_caches=False)
    _check_attention(got, o.out, W.BF16, "grid " + grid)


def test_single_long_sequence_split_over_many_ctas(P):
    wl = W.random_case(78, num_seqs=1, q_lens=[1], ctx_extra=[8191], num_kv_heads=1, group=4, head_dim=128,
                       block_size=16, dtype=W.BF16, max_blocks_per_seq=512)
    b, o, got = _run_both(P, wl, check_caches=False)
    _check_attention(got, o.out, W.BF16, "one sequence")


def test_empty_and_zero_length_query_rows(P):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = W.random_case(5, num_seqs=4, q_lens=[1, 0, 1, 0], ctx_extra=[9, 30, 0, 3], num_kv_heads=2,
                       group=2, head_dim=64, block_size=16, dtype=W.BF16)
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    o = oscen.run(wl, W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry))
    _check_attention(gs.out_as_f64(b.out, W.BF16), o.out, W.BF16)
    assert P.pa_read_device_flags(clear=True) == 0


def test_out_of_range_indices_are_flagged_not_followed(P):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    dev = "cuda"
    geo = W.Geometry(8, 16, 2, 4, 64, W.BF16, 4)
    desc = gs.cache_desc(geo)
    kc = gs.sentinel_cache_dev(geo, dev)
    vc = gs.sentinel_cache_dev(geo, dev)
    k = torch.ones((3, 2, 64), dtype=torch.int16, device=dev)
    slots = torch.tensor([5, 8 * 16, -1], dtype=torch.int32, device=dev)   # middle one is out of range
    P.pa_store_kv(k, k, slots, 3, kc, vc, desc)
    assert P.pa_read_device_flags(clear=True) == P.PA_FLAG_SLOT_RANGE
    bits = gs.cache_bits(kc).reshape(8 * 16, -1)
    assert (bits[5] == 1).all()
    assert (np.delete(bits, 5, axis=0) == W.SENTINEL_BF16).all()
    pairs = torch.tensor([[0, 1], [2, 99]], dtype=torch.int32, device=dev)
    P.pa_copy_blocks(pairs, 2, kc, vc, desc)
    assert P.pa_read_device_flags(clear=True) == P.PA_FLAG_PAIR_RANGE
    q = torch.zeros((2, 4, 64), dtype=torch.int16, device=dev)
    out = torch.zeros_like(q)
    tables = torch.tensor([[0, 77, -1, -1], [1, 2, 3, -1]], dtype=torch.int32, device=dev)
    lens = torch.tensor([20, 70], dtype=torch.int32, device=dev)       # seq 1 exceeds max_context_len
    qsl = torch.tensor([0, 1, 2], dtype=torch.int32, device=dev)
    ws_bytes = P.pa_attention_workspace_size(2, 4, 1, 48, desc)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    P.pa_attention(q, kc, vc, tables, 4, lens, qsl, 2, 2, 4, 1, 48, 0.125, desc, out, ws, stream=None)
    flags = P.pa_read_device_flags(clear=True)
    assert flags & P.PA_FLAG_BLOCK_RANGE and flags & P.PA_FLAG_CONTEXT_RANGE
    assert not flags & P.PA_FLAG_WAIT_TIMEOUT
    assert (out[1] == 0).all()                                         # rows of a rejected sequence untouched


def test_repeated_step_is_idempotent(P):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = W.gqa_long_decode()
    b = gs.prepare(wl)
    gs.run_step(b)
    first = b.out.clone()
    k0 = gs.cache_bits(b.k_cache)
    for _ in range(3):
        gs.run_step(b)
    torch.cuda.synchronize()
    assert torch.equal(first, b.out)
    assert np.array_equal(k0, gs.cache_bits(b.k_cache))


# --------------------------------------------------------------------------
# chunked-prefill rows (tcgen05 path)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["mixed_bs8", "mixed_bs16", "mixed_bs32"])
def test_mixed_config_parity(P, name):
    wl = W.CONFIGS[name]()
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, W.BF16, name)


def _prefill_rows(qsl):
    qsl = np.asarray(qsl)
    return np.concatenate([np.arange(qsl[i], qsl[i + 1]) for i in range(len(qsl) - 1)
                           if qsl[i + 1] - qsl[i] > 1])


def test_mixed_results_agree_across_block_sizes(P):
    """The block size must not change results ([A] §"块大小选择的工程权衡" treats
    it as a tunable). Prefill rows are computed over 128-key tiles at every
    block size, so the same tokens meet the same MMAs in the same tile
    positions and the rows must agree bit for bit; decode rows split their key
    ranges at block boundaries that do depend on the block size, so they agree
    within the attention tolerance."""
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    outs, rows = [], None
    for bs in (8, 16, 32):
        b = gs.prepare(W.mixed_prefill_decode(bs))
        gs.run_step(b)
        torch.cuda.synchronize()
        r = _prefill_rows(b.host["query_start_loc"])
        assert rows is None or np.array_equal(r, rows)
        rows = r
        outs.append(b.out.clone())
        del b
    assert len(rows) == 4 * 256
    idx = torch.as_tensor(rows, device=outs[0].device)
    for o in outs[1:]:
        assert torch.equal(o[idx], outs[0][idx])
    f = [gs.out_as_f64(o, W.BF16) for o in outs]
    assert np.abs(f[0] - f[1]).max() < 2e-2 and np.abs(f[0] - f[2]).max() < 2e-2
    assert P.pa_read_device_flags(clear=True) == 0


def test_mixed_repeated_calls_are_bit_identical(P):
    """Three passes of the mixed step (store + prefill and decode rows) give the
    same output bits: no race between the pipeline stages of either kernel."""
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    b = gs.prepare(W.mixed_prefill_decode(16))
    outs = []
    for _ in range(3):
        b.out.fill_(0)
        gs.run_step(b)
        torch.cuda.synchronize()
        outs.append(b.out.clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    assert P.pa_get_debug_status() == 0


def _random_prefill(seed, d, bs, g, hkv=2):
    q_lens = [2, 37, 130, 1, 64, 1, 200]
    ctx = [0, 100, 517, 30, 0, 1100, 33]
    return W.random_case(seed, num_seqs=len(q_lens), q_lens=q_lens, ctx_extra=ctx, num_kv_heads=hkv,
                         group=g, head_dim=d, block_size=bs, dtype=W.BF16)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("g", [1, 2, 4, 8, 3])
def test_random_prefill_sweep(P, d, bs, g):
    wl = _random_prefill(2000 + d + bs + 11 * g, d, bs, g)
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, W.BF16, "prefill d=%d bs=%d g=%d" % (d, bs, g))


def test_prefill_only_batch_and_full_prompt(P):
    wl = W.random_case(31, num_seqs=3, q_lens=[256, 129, 33], ctx_extra=[0, 0, 1000], num_kv_heads=8,
                       group=4, head_dim=128, block_size=16, dtype=W.BF16)
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, W.BF16, "prefill only")


@pytest.mark.parametrize("q_len,ctx", [(64, 6000), (200, 2500)])
def test_prefill_long_context_split_over_many_ctas(P, q_len, ctx):
    """One prefill chunk on a long context, so few work items of many key
    tiles: (64, 6000) spreads each item over about seven CTAs (the merge's
    general path, more than four pieces), (200, 2500) over three or four."""
    wl = W.random_case(5150 + q_len, num_seqs=2, q_lens=[q_len, 1], ctx_extra=[ctx, 300], num_kv_heads=2,
                       group=4, head_dim=128, block_size=16, dtype=W.BF16)
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, W.BF16, "long-context prefill q_len=%d ctx=%d" % (q_len, ctx))


def test_prefill_large_logits_trigger_rescale(P):
    """Keys scaled so the running max grows tile after tile (exercises the O rescale)."""
    wl = W.random_case(41, num_seqs=2, q_lens=[96, 40], ctx_extra=[700, 300], num_kv_heads=2, group=4,
                       head_dim=128, block_size=16, dtype=W.BF16)
    for op in wl.ops:
        if op.k is not None and op.k.size:
            f = W.bf16_bits_to_f32(op.k)
            ramp = np.linspace(0.5, 6.0, f.shape[0], dtype=np.float32)[:, None, None]
            op.k = W.f32_to_bf16_bits(f * ramp)
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, W.BF16, "rescale")


# --------------------------------------------------------------------------
# grouped-query decode on the tensor cores (bf16, head_dim 128, group 2/4/8)
# --------------------------------------------------------------------------

def test_decode_large_logits_trigger_rescale(P):
    """Keys scaled up along each sequence so the running max keeps growing:
    exercises the lazy rescale of l and of the O^T columns between tiles."""
    wl = _random_decode(4242, W.BF16, 128, 16, 4, hkv=2)
    for op in wl.ops:
        if op.k is not None and op.k.size:
            f = W.bf16_bits_to_f32(op.k)
            ramp = np.linspace(0.5, 8.0, f.shape[0], dtype=np.float32)[:, None, None]
            op.k = W.f32_to_bf16_bits(f * ramp)
    b, o, got = _run_both(P, wl)
    _check_attention(got, o.out, W.BF16, "decode rescale")


def test_decode_many_sequences(P):
    """4600 short sequences: a large per-sequence table in shared memory and
    thousands of units of one or two blocks."""
    rng = np.random.default_rng(4600)
    n = 4600
    lens = rng.integers(1, 48, size=n)
    wl = W.random_case(4600, num_seqs=n, q_lens=[1] * n, ctx_extra=[int(x) - 1 for x in lens], num_kv_heads=1,
                       group=8, head_dim=128, block_size=16, dtype=W.BF16)
    b, o, got = _run_both(P, wl, check_caches=False)
    _check_attention(got, o.out, W.BF16, "many sequences")


@pytest.mark.parametrize("tc", ["0", "1"])
def test_decode_at_the_batch_limit(P, tc):
    """8192 sequences, the largest batch pa_attention takes, on both decode
    kernels (the tensor-core one in a subprocess, since the choice is read once)."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = _LIMIT_SCRIPT
    env = dict(os.environ, PA_DECODE_TC=tc)
    r = subprocess.run([sys.executable, "-c", code, root], capture_output=True, text=True, env=env, cwd=root,
                       timeout=900)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout + r.stderr


_LIMIT_SCRIPT = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from oracle import scenario as oscen
from paged_kv_cache_heads_b200 import workloads as W, scenario as gs
import paged_kv_cache_heads_b200 as P
n = 8192
lens = np.random.default_rng(8192).integers(1, 40, size=n)
wl = W.random_case(8192, num_seqs=n, q_lens=[1] * n, ctx_extra=[int(x) - 1 for x in lens], num_kv_heads=2,
                   group=4, head_dim=128, block_size=16, dtype=W.BF16)
b = gs.prepare(wl)
gs.run_step(b)
torch.cuda.synchronize()
o = oscen.run(wl, W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry))
err = np.abs(gs.out_as_f64(b.out, W.BF16) - o.out)
assert np.isfinite(err).all() and err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
assert P.pa_read_device_flags(clear=True) == 0
print("OK", float(err.max()))
'''


_TENSOR_CORE_SCRIPT = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from oracle import scenario as oscen
from paged_kv_cache_heads_b200 import workloads as W, scenario as gs
import paged_kv_cache_heads_b200 as P
worst = 0.0
cases = []
for seed, g, bs in [(11, 4, 16), (12, 2, 8), (13, 8, 32)]:
    rng = np.random.default_rng(seed)
    lens = [1, bs + 1, int(rng.integers(600, 1400)), int(rng.integers(2000, 2600))]
    wl = W.random_case(seed, num_seqs=4, q_lens=[1] * 4, ctx_extra=[x - 1 for x in lens], num_kv_heads=2,
                       group=g, head_dim=128, block_size=bs, dtype=W.BF16)
    cases.append((seed, wl))
# growing logits (the lazy rescale of l and O^T) and 4600 sequences (whose
# per-sequence table leaves room for only the two-stage ring)
wl = W.random_case(4242, num_seqs=5, q_lens=[1] * 5, ctx_extra=[15, 900, 2500, 40, 1300], num_kv_heads=2, group=4,
                   head_dim=128, block_size=16, dtype=W.BF16)
for op in wl.ops:
    if op.k is not None and op.k.size:
        f = W.bf16_bits_to_f32(op.k)
        op.k = W.f32_to_bf16_bits(f * np.linspace(0.5, 8.0, f.shape[0], dtype=np.float32)[:, None, None])
cases.append(("ramp", wl))
lens = np.random.default_rng(4600).integers(1, 48, size=4600)
cases.append(("many", W.random_case(4600, num_seqs=4600, q_lens=[1] * 4600, ctx_extra=[int(x) - 1 for x in lens],
                                    num_kv_heads=1, group=8, head_dim=128, block_size=16, dtype=W.BF16)))
for seed, wl in cases:
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    o = oscen.run(wl, W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry))
    err = np.abs(gs.out_as_f64(b.out, W.BF16) - o.out)
    assert np.isfinite(err).all() and err.max() <= 2e-2 and err.mean() <= 2e-3, (seed, err.max(), err.mean())
    worst = max(worst, float(err.max()))
assert P.pa_read_device_flags(clear=True) == 0
print("OK", worst)
'''


def test_tensor_core_grouped_decode_matches(P):
    """PA_DECODE_TC=1 selects the tensor-core grouped decode kernel (the
    default is the CUDA-core kernel); it must stay within tolerance too."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PA_DECODE_TC="1")
    r = subprocess.run([sys.executable, "-c", _TENSOR_CORE_SCRIPT, root], capture_output=True, text=True, env=env,
                       cwd=root, timeout=600)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout + r.stderr
