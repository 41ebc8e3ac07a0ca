"""Failure handling on the device, provoked without any fault.

* A bounded wait that runs out: the wait limit is set to 0 for one decode
  call, so the first copy a consumer has to wait for makes it give up. The
  call must report PA_FLAG_WAIT_TIMEOUT, every CTA must wind down (each one
  waits, with the default bound, for the copies it issued before it exits),
  and the next call with the default limit must give the exact bits again.
* Inputs written by the kernel just before the call: attention grids are
  chained to their predecessor (programmatic dependent launch) and must not
  read any input before that predecessor's writes are visible.
"""

import numpy as np
import pytest

from oracle import scenario as oscen
from paged_kv_cache_heads_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_heads_b200 as P
    P.load_library()
    P.pa_read_device_flags(clear=True)
    return P


@pytest.mark.parametrize("name", ["gqa_long", "mixed_bs16"])
def test_bounded_wait_runs_out_and_reports(P, name):
    """gqa_long: decode rows only (the CUDA-core decode grid and the merge);
    mixed_bs16: the prefill grid as well (its MMA, producer and softmax warps
    all give up, then drain their own copies and MMAs before the CTA exits)."""
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    b = gs.prepare(W.CONFIGS[name]())
    gs.run_step(b)
    torch.cuda.synchronize()
    want = b.out.clone()
    assert P.pa_read_device_flags(clear=True) == 0
    prev = P.pa_set_wait_limit_ns(0)
    try:
        gs.run_attention(b)
        torch.cuda.synchronize()
    finally:
        P.pa_set_wait_limit_ns(prev)
    assert prev == 2_000_000_000
    flags = P.pa_read_device_flags(clear=True)
    assert flags == P.PA_FLAG_WAIT_TIMEOUT, hex(flags)
    # the device is still usable, and the next call is exact again
    b.out.fill_(0)
    gs.run_attention(b)
    torch.cuda.synchronize()
    assert torch.equal(b.out, want)
    assert P.pa_get_debug_status() == 0


@pytest.mark.parametrize("name", ["gqa", "mixed"])
def test_index_arrays_written_just_before_the_call_are_seen(P, name):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = (W.random_case(7, num_seqs=6, q_lens=[1, 1, 1, 1, 1, 1], ctx_extra=[900, 15, 2000, 300, 64, 1],
                        num_kv_heads=2, group=4, head_dim=128, block_size=16, dtype=W.BF16) if name == "gqa"
          else W.random_case(8, num_seqs=4, q_lens=[70, 1, 129, 1], ctx_extra=[300, 900, 40, 7],
                             num_kv_heads=2, group=4, head_dim=128, block_size=16, dtype=W.BF16))
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    want = b.out.clone()
    o = oscen.run(wl, W.sentinel_cache(wl.geometry), W.sentinel_cache(wl.geometry))
    err = np.abs(gs.out_as_f64(want, W.BF16) - o.out)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    good_lens = b.context_lens.clone()
    good_qsl = b.query_start_loc.clone()
    for it in range(4):
        # stale values in the arrays, then elementwise torch kernels on the same
        # stream put the right ones back; the last of them runs immediately
        # before the call (context_lens or query_start_loc, alternately)
        b.context_lens.fill_(1)
        b.query_start_loc.zero_()
        b.out.fill_(0)
        torch.cuda.synchronize()
        fixes = [lambda: b.context_lens.add_(good_lens - 1), lambda: b.query_start_loc.add_(good_qsl)]
        for f in (fixes if it % 2 == 0 else fixes[::-1]):
            f()
        gs.run_attention(b)
        torch.cuda.synchronize()
        assert torch.equal(b.out, want)
    assert P.pa_get_debug_status() == 0
