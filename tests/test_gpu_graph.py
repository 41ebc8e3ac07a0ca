"""CUDA-graph capture of the hot-path step (store + attention) through libpa.

The decode step a serving loop repeats every token is captured once and
replayed; replays must give the same output bits as eager calls, and the
result must match the oracle. Mixed batches (prefill + decode rows, whose
attention call chains three kernels) are captured too.
"""

import numpy as np
import pytest

from oracle import scenario as oscen
from paged_kv_cache_heads_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_heads_b200 as P
    P.load_library()
    P.pa_read_device_flags(clear=True)
    return torch


@pytest.mark.parametrize("name", ["gqa_long", "mixed_bs16"])
def test_graph_replay_matches_eager_and_oracle(torch_cuda, name):
    torch = torch_cuda
    import paged_kv_cache_heads_b200 as P
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = W.CONFIGS[name]()
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    eager = b.out.clone()
    b.out.zero_()
    graph = gs.capture_step(b)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(eager, b.out)
    o = oscen.run(wl, W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry))
    err = np.abs(gs.out_as_f64(b.out, W.BF16) - o.out)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert P.pa_read_device_flags(clear=True) == 0


def test_graph_with_host_copies(torch_cuda):
    """The whole e2e step in one graph: pinned-host inputs in, output back out."""
    torch = torch_cuda
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = W.random_case(21, num_seqs=6, q_lens=[1] * 6, ctx_extra=[40, 700, 3, 1200, 16, 90], num_kv_heads=8,
                       group=1, head_dim=128, block_size=16, dtype=W.BF16)
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    want = b.out.cpu()
    q_host = b.q.cpu().pin_memory()
    out_host = torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory()
    b.q.zero_()
    graph = gs.capture_step(b, pre=lambda: b.q.copy_(q_host, non_blocking=True),
                            post=lambda: out_host.copy_(b.out, non_blocking=True))
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out_host, want)


def test_packed_step_inputs_one_copy(torch_cuda):
    """All of a step's inputs staged in one pinned buffer: one host-to-device
    copy, then the usual calls, give the eager result bit for bit."""
    torch = torch_cuda
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = W.CONFIGS["mixed_bs8"]()
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    want = b.out.clone()
    host, dev = gs.pack_step_inputs(b)
    dev.zero_()                                  # nothing left on the device but the caches
    b.out.zero_()
    dev.copy_(host, non_blocking=True)
    gs.run_step(b)
    torch.cuda.synchronize()
    assert torch.equal(b.out, want)
