"""Compaction on the GPU: the block manager remaps held blocks into a dense id
range, pa_copy_blocks moves their K/V data, and attention over the rewritten
tables gives the same output bits as before (nothing in the kernels depends
on which physical blocks hold a sequence)."""

import numpy as np
import pytest

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


@pytest.mark.parametrize("name", ["prefix_cow", "mixed_bs16", "llama7b"])
def test_compaction_preserves_attention_bits(P, name):
    import torch
    from paged_kv_cache_heads_b200 import scenario as gs
    wl = W.CONFIGS[name]()
    b = gs.prepare(wl)
    gs.run_step(b)
    torch.cuda.synchronize()
    want = b.out.clone()
    bm = b.host["bm"]
    held = bm.num_blocks() - bm.num_free()
    pairs = bm.compact()
    assert pairs, "the seeded pools are scattered, so compaction moves blocks"
    assert all(s >= held > d for s, d in pairs)
    dev_pairs = torch.tensor(pairs, dtype=torch.int32, device="cuda")
    P.pa_copy_blocks(dev_pairs, len(pairs), b.k_cache, b.v_cache, b.desc)
    table, lens = bm.block_table(wl.batch_seqs, wl.geometry.max_blocks_per_seq)
    assert table.max() < held
    b.block_tables.copy_(torch.from_numpy(table))
    b.out.zero_()
    gs.run_attention(b)
    torch.cuda.synchronize()
    assert torch.equal(b.out, want)
    assert P.pa_read_device_flags(clear=True) == 0
