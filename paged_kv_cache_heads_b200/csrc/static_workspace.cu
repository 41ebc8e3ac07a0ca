// pa_attention_static_workspace: pa_attention for callers that cannot allocate
// device memory.
//
// pa_attention takes its split-K scratch (per-split partial outputs and their
// log-sum-exp) from a caller-provided workspace. Some callers have no way to
// provide one: a serving process whose device memory is handed out entirely
// by its own pool, a plug-in host that does not let a library touch the CUDA
// allocator, or a latency-critical loop that must not call cudaMalloc /
// cudaFree because they can synchronise the whole device. This entry point
// gives them the same computation with the scratch held in a fixed array that
// is part of this library's device image: no allocation happens in any call.
//
// Cost: the array (PA_STATIC_WORKSPACE_BYTES) occupies device memory on every
// GPU that loads the library, until the process exits.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace {

// Split-K scratch shared by every call of pa_attention_static_workspace.
static __device__ __align__(256) unsigned char g_attention_scratch[PA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_attention_scratch on the current device. In host code
// the array's name only stands in for the symbol, so the address must come
// from cudaGetSymbolAddress, once per device, with that device current.
cudaError_t scratch_address(void** out) {
  static void* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attention_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" pa_status pa_attention_static_workspace(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    int32_t max_blocks_per_seq, const int32_t* context_lens, const int32_t* query_start_loc,
    int32_t num_seqs, int32_t num_q_tokens, int32_t num_q_heads, int32_t max_query_len,
    int32_t max_context_len, float scale, const pa_cache_desc* cache, void* out, void* stream) {
  const size_t need =
      pa_attention_workspace_size(num_seqs, num_q_heads, max_query_len, max_context_len, cache);
  if (need > PA_STATIC_WORKSPACE_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "pa_attention_static_workspace: this batch needs %zu bytes of scratch, more than the "
             "fixed %u bytes (use pa_attention with a caller workspace, or split the batch)",
             need, static_cast<unsigned>(PA_STATIC_WORKSPACE_BYTES));
    pa::set_last_error(msg);
    return PA_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_address(&ws);
    if (e != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof(msg), "pa_attention_static_workspace: cudaGetSymbolAddress: %s",
               cudaGetErrorString(e));
      pa::set_last_error(msg);
      return PA_ERR_CUDA;
    }
  }
  // Nothing in the scratch has to start at zero: every split writes its
  // partial before the merge reads it, so stale contents of an earlier call
  // are never used.
  return pa_attention(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, query_start_loc,
                      num_seqs, num_q_tokens, num_q_heads, max_query_len, max_context_len, scale, cache, out,
                      ws, need > 0 ? size_t(PA_STATIC_WORKSPACE_BYTES) : size_t(0), stream);
}
