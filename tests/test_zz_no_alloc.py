"""pa_attention_static_workspace: attention without a caller workspace.

The entry point serves callers that cannot allocate device memory (a process
whose device memory is handed out entirely by its own pool, a host framework
that keeps libraries away from the CUDA allocator, a loop that must not call
cudaMalloc/cudaFree). Its split-K scratch is a fixed array inside libpa.

Checked through the C ABI: two calls in a row on different batches (the
second sees the scratch the first left behind) give the same output bits as
pa_attention with a caller workspace -- both run the same kernels on the same
grid and differ only in where the scratch lives, so any read of stale scratch
would show up as a changed bit -- and stay within the attention tolerance of
the fp64 oracle; a batch needing more scratch than the array is rejected.
This file is named so that pytest collects it last.
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
    return P


def _static_call(P, b, out):
    geo = b.wl.geometry
    P.pa_attention_static_workspace(b.q, b.k_cache, b.v_cache, b.block_tables, geo.max_blocks_per_seq,
                                    b.context_lens, b.query_start_loc, len(b.wl.batch_seqs), b.wl.num_q_tokens,
                                    geo.num_q_heads, b.wl.max_query_len, b.max_context_len, b.wl.scale, b.desc,
                                    out)


def test_static_workspace_matches_caller_workspace_on_two_calls(P):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    batches = [
        gs.prepare(W.gqa_long_decode()),                     # long sequences, many splits
        gs.prepare(W.random_case(9, num_seqs=5, q_lens=[1, 40, 1, 1, 3], ctx_extra=[2500, 300, 15, 900, 0],
                                 num_kv_heads=2, group=4, head_dim=128, block_size=16, dtype=W.BF16)),
    ]
    for b in batches:
        assert b.workspace is not None                       # these batches do use split-K scratch
        gs.run_step(b)                                       # store + pa_attention with its workspace
        want = b.out.clone()
        got = torch.full_like(b.out, 0x7FC1)
        _static_call(P, b, got)
        torch.cuda.synchronize()
        assert torch.equal(got, want)                        # bit for bit: same kernels, same grid
        o = oscen.run(b.wl, W.sentinel_cache(b.wl.geometry), W.sentinel_cache(b.wl.geometry))
        g = gs.out_as_f64(got, W.BF16)
        err = np.abs(g - o.out)
        assert np.isfinite(g).all()
        assert err.max() <= AMAX and err.mean() <= AMEAN, (err.max(), err.mean())
    assert P.pa_read_device_flags(clear=True) == 0


def test_static_workspace_rejects_batches_beyond_its_size(P):
    import torch
    desc = (1 << 20, 16, 32, 128, P.PA_BF16)
    need = P.pa_attention_workspace_size(4096, 32, 1, 16384, desc)
    assert need > P.PA_STATIC_WORKSPACE_BYTES
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(P.PAError) as e:
        P.pa_attention_static_workspace(t, t, t, t, 1024, t, t, 4096, 4096, 32, 1, 16384, 0.088, desc, t)
    assert e.value.status == P.PA_ERR_UNSUPPORTED and "scratch" in str(e.value)
