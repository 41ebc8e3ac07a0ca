// Host block manager: free list, per-sequence block tables, reference counts
// and copy-on-write. Produces int32 index arrays only; never touches a GPU.
//
// Rules restated from the pages:
//  * "深入剖析nano-vLLM推理引擎架构：PagedAttention内存管理实现",
//    §"PagedAttention：操作系统的内存智慧": the pool is a list of free physical
//    blocks; each sequence has a table from logical to physical blocks; a new
//    block is taken only when the sequence's current block is full.
//  * same page, §"连续批处理与内存管理的协同": a finished request returns all of
//    its blocks to the free list at once.
//  * "vLLM核心架构：PagedAttention原理、KV Cache管理、连续批处理机制",
//    §"二、KV Cache管理：从浪费到极致复用": requests with a common prefix point
//    at the same pages; reference counts decide when a page is really free;
//    a shared page is copied only when one of its holders writes into it.
// Choices the pages leave open: the free list is FIFO (take from the front,
// return to the back) from a caller-given initial order; a call that needs
// more blocks than are free fails before changing anything; freed blocks
// return in logical order; a write copies the shared last block only when
// that block is partly filled (a full block is never written again).
#include <algorithm>
#include <chrono>
#include <cstdint>
#include <cstdio>
#include <deque>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include "pa.h"
#include "pa_internal.h"

namespace {

pa_status bm_fail(pa_status st, const char* msg) {
  pa::set_last_error(msg);
  return st;
}

struct Sequence {
  std::vector<int32_t> blocks;
  int32_t len = 0;
};

int32_t blocks_for(int64_t tokens, int32_t bs) { return static_cast<int32_t>((tokens + bs - 1) / bs); }

}  // namespace

struct pa_bm {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::deque<int32_t> free_list;
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Sequence> seqs;
  // latency of block-allocating calls, last kLatencyWindow samples (microseconds)
  static constexpr size_t kLatencyWindow = 4096;
  std::vector<float> latency_us;
  size_t latency_next = 0;
  int64_t latency_count = 0;

  void record_latency(std::chrono::steady_clock::time_point t0) {
    const float us = std::chrono::duration<float, std::micro>(std::chrono::steady_clock::now() - t0).count();
    if (latency_us.size() < kLatencyWindow) {
      latency_us.push_back(us);
    } else {
      latency_us[latency_next] = us;
    }
    latency_next = (latency_next + 1) % kLatencyWindow;
    ++latency_count;
  }

  int32_t take() {
    const int32_t b = free_list.front();
    free_list.pop_front();
    ref[b] = 1;
    return b;
  }
};

extern "C" {

pa_status pa_bm_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_free_order,
                       pa_bm** out) {
  if (!out) return bm_fail(PA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (num_blocks < 0 || block_size < 1) return bm_fail(PA_ERR_INVALID_ARG, "bad pool geometry");
  pa_bm* bm = new (std::nothrow) pa_bm;
  if (!bm) return bm_fail(PA_ERR_INVALID_ARG, "out of host memory");
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref.assign(num_blocks, 0);
  if (initial_free_order) {
    std::vector<uint8_t> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      const int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return bm_fail(PA_ERR_INVALID_ARG, "initial_free_order is not a permutation of the pool");
      }
      seen[b] = 1;
      bm->free_list.push_back(b);
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) bm->free_list.push_back(i);
  }
  *out = bm;
  return PA_OK;
}

void pa_bm_destroy(pa_bm* bm) { delete bm; }

pa_status pa_bm_slot_mapping(const pa_bm* bm, int64_t seq_id, int32_t start, int32_t n, int32_t* out) {
  if (!bm) return bm_fail(PA_ERR_INVALID_ARG, "bm is NULL");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return bm_fail(PA_ERR_INDEX, "unknown sequence");
  if (start < 0 || n < 0 || int64_t(start) + n > it->second.len)
    return bm_fail(PA_ERR_INDEX, "positions outside the sequence");
  if (n > 0 && !out) return bm_fail(PA_ERR_INVALID_ARG, "out is NULL");
  const auto& blocks = it->second.blocks;
  const int32_t bs = bm->block_size;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t p = start + i;
    out[i] = blocks[p / bs] * bs + p % bs;
  }
  return PA_OK;
}

pa_status pa_bm_add_seq(pa_bm* bm, int64_t seq_id, int32_t num_tokens, int32_t* slots_out) {
  if (!bm) return bm_fail(PA_ERR_INVALID_ARG, "bm is NULL");
  const auto t0 = std::chrono::steady_clock::now();
  if (num_tokens < 0) return bm_fail(PA_ERR_INVALID_ARG, "num_tokens < 0");
  if (bm->seqs.count(seq_id)) return bm_fail(PA_ERR_INVALID_ARG, "sequence already exists");
  const int32_t need = blocks_for(num_tokens, bm->block_size);
  if (need > static_cast<int32_t>(bm->free_list.size()))
    return bm_fail(PA_ERR_OUT_OF_BLOCKS, "not enough free blocks");
  Sequence seq;
  seq.blocks.reserve(need);
  for (int32_t i = 0; i < need; ++i) seq.blocks.push_back(bm->take());
  seq.len = num_tokens;
  bm->seqs.emplace(seq_id, std::move(seq));
  bm->record_latency(t0);
  if (slots_out) return pa_bm_slot_mapping(bm, seq_id, 0, num_tokens, slots_out);
  return PA_OK;
}

pa_status pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child, int32_t num_tokens) {
  if (!bm) return bm_fail(PA_ERR_INVALID_ARG, "bm is NULL");
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end()) return bm_fail(PA_ERR_INDEX, "unknown parent sequence");
  if (bm->seqs.count(child)) return bm_fail(PA_ERR_INVALID_ARG, "child sequence already exists");
  const int32_t n = num_tokens < 0 ? it->second.len : num_tokens;
  if (n > it->second.len) return bm_fail(PA_ERR_INDEX, "fork longer than the parent");
  Sequence seq;
  const int32_t nb = blocks_for(n, bm->block_size);
  seq.blocks.assign(it->second.blocks.begin(), it->second.blocks.begin() + nb);
  for (int32_t b : seq.blocks) ++bm->ref[b];
  seq.len = n;
  bm->seqs.emplace(child, std::move(seq));
  return PA_OK;
}

pa_status pa_bm_append_tokens(pa_bm* bm, int64_t seq_id, int32_t n, int32_t* slots_out,
                              int32_t* cow_pair_out, int32_t* num_cow_out) {
  if (!bm) return bm_fail(PA_ERR_INVALID_ARG, "bm is NULL");
  if (n < 0) return bm_fail(PA_ERR_INVALID_ARG, "n < 0");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return bm_fail(PA_ERR_INDEX, "unknown sequence");
  const auto t0 = std::chrono::steady_clock::now();
  Sequence& seq = it->second;
  const int32_t bs = bm->block_size;
  if (int64_t(seq.len) + n > INT32_MAX) return bm_fail(PA_ERR_INVALID_ARG, "sequence too long");
  const bool cow = n > 0 && seq.len % bs != 0 && bm->ref[seq.blocks.back()] > 1;
  const int32_t need = blocks_for(int64_t(seq.len) + n, bs) - blocks_for(seq.len, bs) + (cow ? 1 : 0);
  if (need > static_cast<int32_t>(bm->free_list.size()))
    return bm_fail(PA_ERR_OUT_OF_BLOCKS, "not enough free blocks");
  if (num_cow_out) *num_cow_out = 0;
  if (cow) {
    const int32_t old_block = seq.blocks.back();
    const int32_t new_block = bm->take();
    --bm->ref[old_block];
    seq.blocks.back() = new_block;
    if (cow_pair_out) {
      cow_pair_out[0] = old_block;
      cow_pair_out[1] = new_block;
    }
    if (num_cow_out) *num_cow_out = 1;
  }
  for (int32_t i = 0; i < n; ++i) {
    const int32_t p = seq.len + i;
    if (p % bs == 0) seq.blocks.push_back(bm->take());
    if (slots_out) slots_out[i] = seq.blocks[p / bs] * bs + p % bs;
  }
  seq.len += n;
  bm->record_latency(t0);
  return PA_OK;
}

pa_status pa_bm_free_seq(pa_bm* bm, int64_t seq_id) {
  if (!bm) return bm_fail(PA_ERR_INVALID_ARG, "bm is NULL");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return bm_fail(PA_ERR_INDEX, "unknown sequence");
  for (int32_t b : it->second.blocks)
    if (--bm->ref[b] == 0) bm->free_list.push_back(b);
  bm->seqs.erase(it);
  return PA_OK;
}

pa_status pa_bm_block_table(const pa_bm* bm, const int64_t* seq_ids, int32_t n, int32_t max_blocks,
                            int32_t* table_out, int32_t* ctx_lens_out) {
  if (!bm) return bm_fail(PA_ERR_INVALID_ARG, "bm is NULL");
  if (n < 0 || max_blocks < 0) return bm_fail(PA_ERR_INVALID_ARG, "negative size");
  if (n > 0 && (!seq_ids || (max_blocks > 0 && !table_out)))
    return bm_fail(PA_ERR_INVALID_ARG, "NULL output");
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return bm_fail(PA_ERR_INDEX, "unknown sequence");
    if (static_cast<int32_t>(it->second.blocks.size()) > max_blocks)
      return bm_fail(PA_ERR_INVALID_ARG, "sequence holds more than max_blocks blocks");
  }
  for (int32_t i = 0; i < n; ++i) {
    const Sequence& seq = bm->seqs.find(seq_ids[i])->second;
    int32_t* row = table_out + static_cast<size_t>(i) * max_blocks;
    const int32_t nb = static_cast<int32_t>(seq.blocks.size());
    for (int32_t j = 0; j < max_blocks; ++j) row[j] = j < nb ? seq.blocks[j] : -1;
    if (ctx_lens_out) ctx_lens_out[i] = seq.len;
  }
  return PA_OK;
}

int32_t pa_bm_num_free(const pa_bm* bm) { return bm ? static_cast<int32_t>(bm->free_list.size()) : -1; }

int32_t pa_bm_num_blocks(const pa_bm* bm) { return bm ? bm->num_blocks : -1; }

int32_t pa_bm_refcount(const pa_bm* bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  return bm->ref[block];
}

int32_t pa_bm_seq_len(const pa_bm* bm, int64_t seq_id) {
  if (!bm) return -1;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? -1 : it->second.len;
}

pa_status pa_bm_cascade_groups(const pa_bm* bm, const int64_t* seq_ids, int32_t n, int32_t min_shared_blocks,
                               int32_t* shared_out, int32_t* groups_out, int32_t* num_groups_out) {
  if (!bm || n < 0 || min_shared_blocks < 1 || !num_groups_out || (n > 0 && (!seq_ids || !shared_out || !groups_out)))
    return bm_fail(PA_ERR_INVALID_ARG, "bad cascade_groups arguments");
  std::vector<const Sequence*> seq(n);
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return bm_fail(PA_ERR_INDEX, "unknown sequence");
    seq[i] = &it->second;
    shared_out[i] = 0;
  }
  auto full_blocks = [&](int32_t i) { return seq[i]->len / bm->block_size; };
  int32_t groups = 0, i = 0;
  while (i < n) {
    // extend [i, j) while the members still share >= min_shared_blocks full leading blocks
    int32_t common = full_blocks(i), j = i + 1;
    while (j < n) {
      const int32_t c = std::min(common, full_blocks(j));
      int32_t k = 0;
      while (k < c && seq[j]->blocks[k] == seq[i]->blocks[k]) ++k;
      if (k < min_shared_blocks) break;
      common = k;
      ++j;
    }
    if (j - i >= 2 && common >= min_shared_blocks) {
      groups_out[2 * groups] = i;
      groups_out[2 * groups + 1] = j - i;
      ++groups;
      for (int32_t m = i; m < j; ++m) shared_out[m] = common;
      i = j;
    } else {
      ++i;
    }
  }
  *num_groups_out = groups;
  return PA_OK;
}

pa_status pa_bm_compact(pa_bm* bm, int32_t* pairs_out, int32_t cap, int32_t* num_pairs_out) {
  if (!bm || !num_pairs_out) return bm_fail(PA_ERR_INVALID_ARG, "NULL argument");
  if (cap < 0) return bm_fail(PA_ERR_INVALID_ARG, "negative capacity");
  int32_t held = 0;
  for (int32_t b = 0; b < bm->num_blocks; ++b) held += bm->ref[b] > 0;
  // movers: held blocks at or past `held`; holes: free ids below it (both ascending)
  std::vector<int32_t> map(bm->num_blocks);
  for (int32_t b = 0; b < bm->num_blocks; ++b) map[b] = b;
  int32_t n = 0, hole = 0;
  for (int32_t b = held; b < bm->num_blocks; ++b) {
    if (bm->ref[b] == 0) continue;
    while (bm->ref[hole] > 0) ++hole;  // a hole exists below `held` for every mover
    map[b] = hole++;
    ++n;
  }
  *num_pairs_out = n;
  if (n > cap || (n > 0 && !pairs_out)) return bm_fail(PA_ERR_INVALID_ARG, "pairs_out holds fewer than the moves");
  int32_t k = 0;
  for (int32_t b = held; b < bm->num_blocks; ++b) {
    if (map[b] == b) continue;
    pairs_out[2 * k] = b;
    pairs_out[2 * k + 1] = map[b];
    ++k;
    bm->ref[map[b]] = bm->ref[b];
    bm->ref[b] = 0;
  }
  for (auto& kv : bm->seqs)
    for (int32_t& b : kv.second.blocks) b = map[b];
  bm->free_list.clear();
  for (int32_t b = held; b < bm->num_blocks; ++b) bm->free_list.push_back(b);
  return PA_OK;
}

pa_status pa_bm_get_stats(const pa_bm* bm, double kv_bytes_per_block, pa_bm_stats* out) {
  if (!bm || !out) return bm_fail(PA_ERR_INVALID_ARG, "NULL argument");
  pa_bm_stats st = {};
  const int32_t bs = bm->block_size;
  st.num_blocks = bm->num_blocks;
  st.free_blocks = static_cast<int32_t>(bm->free_list.size());
  st.num_seqs = static_cast<int32_t>(bm->seqs.size());
  // tokens a held block holds: the most any of its holders has written into it
  std::vector<int32_t> fill(bm->num_blocks, 0);
  for (const auto& kv : bm->seqs) {
    const Sequence& seq = kv.second;
    st.logical_blocks += static_cast<int64_t>(seq.blocks.size());
    st.tokens += seq.len;
    for (size_t i = 0; i < seq.blocks.size(); ++i) {
      const int64_t in_block = std::min<int64_t>(bs, int64_t(seq.len) - int64_t(i) * bs);
      fill[seq.blocks[i]] = std::max<int32_t>(fill[seq.blocks[i]], static_cast<int32_t>(in_block));
    }
  }
  for (int32_t b = 0; b < bm->num_blocks; ++b)
    if (bm->ref[b] > 0) {
      ++st.held_blocks;
      st.used_slots += fill[b];
    }
  st.block_utilisation = bm->num_blocks ? double(st.held_blocks) / bm->num_blocks : 0.0;
  st.internal_fragmentation = st.held_blocks ? 1.0 - double(st.used_slots) / (double(st.held_blocks) * bs) : 0.0;
  st.sharing_saving = st.logical_blocks ? 1.0 - double(st.held_blocks) / double(st.logical_blocks) : 0.0;
  st.table_bytes = 4.0 * double(st.logical_blocks);
  st.table_overhead = (bm->num_blocks && kv_bytes_per_block > 0)
                          ? st.table_bytes / (double(bm->num_blocks) * kv_bytes_per_block)
                          : 0.0;
  if (!bm->latency_us.empty()) {
    std::vector<float> v(bm->latency_us);
    std::sort(v.begin(), v.end());
    auto pct = [&](double q) { return double(v[std::min(v.size() - 1, size_t(q * (v.size() - 1) + 0.5))]); };
    st.alloc_p50_us = pct(0.50);
    st.alloc_p99_us = pct(0.99);
  }
  st.alloc_samples = bm->latency_count;
  *out = st;
  return PA_OK;
}

int32_t pa_bm_free_list(const pa_bm* bm, int32_t* out, int32_t cap) {
  if (!bm || cap < 0 || (cap > 0 && !out)) return -1;
  int32_t i = 0;
  for (auto it = bm->free_list.begin(); it != bm->free_list.end() && i < cap; ++it) out[i++] = *it;
  return i;
}

}  // extern "C"
