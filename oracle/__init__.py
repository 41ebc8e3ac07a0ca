"""Oracle for the paged KV-cache hot path: TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct CPU restatement (NumPy, float64) of what the
CUDA library computes. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The
product path (``paged_kv_cache_heads_b200``) never imports, calls or links
anything here, and nothing here imports the product.

Pages restated (titles as published; sections as headed on each page):
  [A] "深入剖析nano-vLLM推理引擎架构：PagedAttention内存管理实现"
      (blog.hotdry.top, 2026-02-02)
  [B] "深入解析 nano-vLLM 推理引擎的分页 KV 缓存与内存优化架构"
      (blog.hotdry.top, 2026-02-02)
  [C] "vLLM核心架构：PagedAttention原理、KV Cache管理、连续批处理机制"

Pin status of every public function: see the docstring of each; all are
pinned by ``tests/test_oracle_pins.py`` and ``tests/test_oracle_block_manager.py``.
"""

from .paged_kv import (  # noqa: F401
    BlockManager,
    OutOfBlocks,
    as_f64,
    copy_blocks,
    kv_bytes_per_token,
    paged_attention,
    paged_attention_bruteforce,
    preallocation_fragmentation,
    slot_of,
    store_kv,
    store_kv_bruteforce,
)
