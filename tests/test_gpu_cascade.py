"""Cascade (shared-prefix) decode on the GPU against the oracle.

pa_attention_cascade computes the same attention as pa_attention; it only
reads each group's shared blocks once. Its output is compared with the fp64
oracle over the full sequences (tolerance of the bf16 parity tests) and with
pa_attention on the same batch, on the shared-prompt configuration and on
random batches that mix groups with unshared sequences.
"""

import numpy as np
import pytest

from oracle import scenario as oscen
from paged_kv_cache_heads_b200 import workloads as W

pytestmark = pytest.mark.gpu

AMAX, AMEAN = 2e-2, 2e-3


@pytest.fixture(scope="module")
def P():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_heads_b200 as P
    P.load_library()
    P.pa_read_device_flags(clear=True)
    return P


def _check(got, ref, ctx):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), ctx
    assert err.max() <= AMAX and err.mean() <= AMEAN, (ctx, err.max(), err.mean())


def _run(P, wl, min_shared_blocks=1, expect_groups=True):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    b = gs.prepare(wl)
    gs.run_step(b)                       # store the step's rows + plain attention
    plan = gs.plan_cascade(b, min_shared_blocks)
    if expect_groups:
        assert plan.num_groups > 0
    out = torch.full_like(b.out, 0x7FC1)
    gs.run_attention_cascade(b, plan, out=out)
    torch.cuda.synchronize()
    assert P.pa_read_device_flags(clear=True) == 0
    o = oscen.run(wl, W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry))
    got = gs.out_as_f64(out, wl.geometry.dtype)
    plain = gs.out_as_f64(b.out, wl.geometry.dtype)
    return got, plain, o.out, plan


def test_cascade_shared_prompt_config(P):
    wl = W.prefix_cow_decode()
    got, plain, ref, plan = _run(P, wl)
    assert plan.num_groups == 1 and plan.max_shared_blocks == 124
    _check(got, ref, "prefix_cow cascade")
    _check(got, plain, "prefix_cow cascade vs pa_attention")


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("g,d", [(4, 128), (1, 128), (8, 64), (2, 128)])
def test_cascade_random_groups(P, bs, g, d):
    rng = np.random.default_rng(70 + bs + 3 * g + d)
    groups = [
        (int(rng.integers(300, 700)), [0] * 3),                  # several 256-token prefix chunks
        (int(rng.integers(bs, 3 * bs)), [0] * 2),               # a short prefix, two members
        (int(rng.integers(40, 200)), [0] * 37),                 # more members than one 32-row tile
    ]
    groups = [(p, [p + int(rng.integers(1, 300)) for _ in m]) for p, m in groups]
    singles = [int(rng.integers(1, 900)) for _ in range(3)]
    wl = W.shared_prefix_case(500 + bs + g + d, groups=groups, singles=singles, num_kv_heads=2, group=g,
                              head_dim=d, block_size=bs, dtype=W.BF16)
    got, plain, ref, plan = _run(P, wl)
    _check(got, ref, "bs=%d g=%d d=%d" % (bs, g, d))


def test_cascade_without_groups_equals_plain_decode(P):
    wl = W.random_case(12, num_seqs=6, q_lens=[1] * 6, ctx_extra=[3, 100, 900, 17, 2000, 64], num_kv_heads=2,
                       group=4, head_dim=128, block_size=16, dtype=W.BF16)
    got, plain, ref, plan = _run(P, wl, expect_groups=False)
    assert plan.num_groups == 0
    _check(got, ref, "no groups")


def test_cascade_member_with_no_own_blocks(P):
    """Two sequences that share every block (lengths a multiple of the block
    size, identical tables): the decode pass streams nothing for them and the
    merge takes the prefix pass alone."""
    import torch
    import paged_kv_cache_heads_b200 as PP
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = W.random_case(13, num_seqs=3, q_lens=[1] * 3, ctx_extra=[255, 40, 700], num_kv_heads=2, group=4,
                       head_dim=128, block_size=16, dtype=W.BF16)
    b = gs.prepare(wl)
    gs.run_step(b)
    # sequence 1 reads sequence 0's blocks and length (256 tokens = 16 full blocks)
    b.block_tables[1].copy_(b.block_tables[0])
    b.context_lens[1].copy_(b.context_lens[0])
    gs.run_attention(b)
    want = b.out.clone()
    shared = torch.tensor([16, 16, 0], dtype=torch.int32, device="cuda")
    groups = torch.tensor([[0, 2]], dtype=torch.int32, device="cuda")
    geo = wl.geometry
    ws_b = PP.pa_attention_cascade_workspace_size(3, geo.num_q_heads, b.max_context_len, 16, b.desc)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    out = torch.full_like(b.out, 0x7FC1)
    PP.pa_attention_cascade(b.q, b.k_cache, b.v_cache, b.block_tables, geo.max_blocks_per_seq, b.context_lens,
                            b.query_start_loc, 3, geo.num_q_heads, b.max_context_len, shared, groups, 1, 2, 16,
                            wl.scale, b.desc, out, ws)
    torch.cuda.synchronize()
    assert P.pa_read_device_flags(clear=True) == 0
    _check(gs.out_as_f64(out, W.BF16), gs.out_as_f64(want, W.BF16), "all blocks shared")


def test_cascade_graph_replay(P):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = W.prefix_cow_decode()
    b = gs.prepare(wl)
    gs.run_step(b)
    plan = gs.plan_cascade(b)
    gs.run_attention_cascade(b, plan)
    torch.cuda.synchronize()
    eager = b.out.clone()
    b.out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gs.run_attention_cascade(b, plan)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(eager, b.out)
    assert P.pa_read_device_flags(clear=True) == 0


_FORCED_TC_SCRIPT = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from oracle import scenario as oscen
from paged_kv_cache_heads_b200 import workloads as W, scenario as gs
import paged_kv_cache_heads_b200 as P
for seed, g, bs in [(31, 4, 16), (32, 8, 8), (33, 2, 32)]:
    rng = np.random.default_rng(seed)
    groups = [(int(rng.integers(300, 700)), [0] * 3), (int(rng.integers(40, 200)), [0] * 37)]
    groups = [(p, [p + int(rng.integers(1, 300)) for _ in m]) for p, m in groups]
    wl = W.shared_prefix_case(seed, groups=groups, singles=[17, 700], num_kv_heads=2, group=g, head_dim=128,
                              block_size=bs, dtype=W.BF16)
    b = gs.prepare(wl)
    gs.run_step(b)
    plan = gs.plan_cascade(b)
    out = torch.zeros_like(b.out)
    gs.run_attention_cascade(b, plan, out=out)
    torch.cuda.synchronize()
    o = oscen.run(wl, W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry))
    err = np.abs(gs.out_as_f64(out, W.BF16) - o.out)
    assert np.isfinite(err).all() and err.max() <= 2e-2 and err.mean() <= 2e-3, (seed, err.max(), err.mean())
assert P.pa_read_device_flags(clear=True) == 0
print("OK")
'''


def test_cascade_with_tensor_core_suffix_pass(P):
    """The suffix pass runs on the CUDA-core kernel by default (short units);
    PA_DECODE_TC=1 forces the tensor-core kernel, whose skipping of shared
    blocks must give the same results."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PA_DECODE_TC="1")
    r = subprocess.run([sys.executable, "-c", _FORCED_TC_SCRIPT, root], capture_output=True, text=True, env=env,
                       cwd=root, timeout=600)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout + r.stderr
