// Internal launcher interface between the C-ABI layer (pa_api.cu) and the
// kernel translation units. Host code only; no torch types anywhere.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"

#ifndef PA_WAIT_LIMIT_NS
#define PA_WAIT_LIMIT_NS 2000000000ull  // default bound of a device-side wait: 2 s
#endif

namespace pa {

// Device-side work description of one pa_attention call (decode part).
struct DecodeArgs {
  const void* q;
  void* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start_loc;
  float* part_o;        // [slots][GH][head_dim] fp32 partial outputs
  float* part_lse;      // [slots][GH] fp32 log2-sum-exp of each partial
  int32_t* seq_prefix;  // [num_seqs + 1] decode blocks before each sequence
  unsigned* status;     // library status word
  int32_t max_blocks_per_seq;
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t num_blocks;
  int32_t max_context_len;
  int32_t grid;         // CTAs of the decode grid (set by the decode launcher)
  int32_t hpu;          // query heads per unit of the decode grid (set by the decode launcher)
  float scale_log2;     // scale * log2(e)
  uint64_t wait_limit_ns;  // bound of every device-side wait on another party (pa_set_wait_limit_ns)
  // Cascade (shared-prefix) decode; all null / 0 otherwise.
  const int32_t* skip_blocks;  // [num_seqs] leading table blocks read by the prefix pass instead
  const float* l1_o;           // [num_seqs * num_q_heads * l1_max_chunks][head_dim] prefix-pass partials
  const float* l1_lse;         // [num_seqs * num_q_heads * l1_max_chunks]
  int32_t l1_max_chunks;       // prefix chunks per sequence and head (slot stride)
  int32_t l1_chunk_blocks;     // blocks per prefix chunk
};

struct PrefillArgs {
  const void* k_cache;  // [num_blocks][block_size][num_kv_heads][head_dim]
  const void* v_cache;
  void* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start_loc;
  unsigned* status;
  int32_t max_blocks_per_seq;
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t num_blocks;
  int32_t max_context_len;
  int32_t max_query_len;
  int32_t num_q_tokens;
  float scale_log2;
  uint64_t wait_limit_ns;  // bound of every device-side wait on another party (pa_set_wait_limit_ns)
  // Cascade prefix pass (kernel instantiated with the cascade flag): work
  // items run over the groups' shared blocks instead of the prefill rows.
  const int32_t* groups;       // [num_groups][2]: first member sequence, member count
  const int32_t* skip_blocks;  // [num_seqs] shared blocks of each member (same within a group)
  int32_t num_groups;
  float* l1_o;                 // partial outputs, slot ((s * num_q_heads + h) * l1_max_chunks + chunk)
  float* l1_lse;
  int32_t l1_max_chunks;
  int32_t l1_chunk_blocks;
  // Prefill rows (workspace): per CTA, the work item it starts and the next
  // CTAs continue ([grid]: first query row, rows left in the sequence, first
  // query head, last covering CTA or -1), written by the kernel for the merge;
  // partials of split work items, two slots per CTA of 256 rows each
  // ([2 * grid][256][head_dim] fp16 and [2 * grid][256] fp32).
  int4* pf_split;
  uint16_t* pf_o;               // partial O / l rows as IEEE fp16 bits
  float* pf_lse;
  int32_t grid;                // CTAs of the prefill grid (prefill_grid)
};

// CTAs of the prefill grid for a call with these host bounds: one per SM,
// fewer when the call cannot have 8 key tiles of work per CTA. The workspace
// holds two partial slots per CTA.
int32_t prefill_grid(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_query_len,
                     int32_t max_context_len);

// Sets the calling thread's pa_last_error() message.
void set_last_error(const char* msg);

// Current bound of the kernels' device-side waits (pa_set_wait_limit_ns).
uint64_t wait_limit_ns();

// Upper bound on the decode grid; the workspace holds S*Hq/GH + this many partial slots.
int32_t decode_max_grid();
inline int32_t ceil_div(int64_t a, int64_t b) { return static_cast<int32_t>((a + b - 1) / b); }

// Launchers return cudaSuccess or the launch error. `maps` are encoded tensor
// maps for the K and V caches (box and swizzle as the kernel requires).
cudaError_t launch_store_kv(const void* k, const void* v, const int32_t* slots, int32_t num_tokens,
                            void* k_cache, void* v_cache, const pa_cache_desc& c, unsigned* status,
                            cudaStream_t stream);
cudaError_t launch_copy_blocks(const int32_t* pairs, int32_t num_pairs, void* k_cache,
                               void* v_cache, const pa_cache_desc& c, unsigned* status,
                               cudaStream_t stream);
cudaError_t launch_decode(DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          const pa_cache_desc& c, cudaStream_t stream);
// Grouped-query decode on the tensor cores: bf16, head_dim 128, group 2, 4 or 8,
// selected only with environment PA_DECODE_TC=1. Decode runs on the CUDA-core
// kernel by default: the tensor cores are kept for the dense contractions of
// prefill and the cascade prefix pass, and with chained launches the CUDA-core
// grouped kernel matches the tensor-core one on the grouped batches measured
// (within 5 %, faster on two of three). `short_units` marks the cascade suffix
// pass (units of a few blocks), where the CUDA-core kernel is also the better fit.
// `qmap` is q as {head_dim, num_q_heads, num_q_tokens} with box {64, group, 1};
// the cache maps have box {64, 1, block_size, 1}; all three use the 128-byte swizzle.
bool decode_tc_supported(int32_t group, const pa_cache_desc& c);
bool decode_uses_tc(int32_t group, const pa_cache_desc& c, bool short_units);
cudaError_t launch_decode_tc(DecodeArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, const pa_cache_desc& c, cudaStream_t stream);
cudaError_t launch_decode_combine(const DecodeArgs& a, const pa_cache_desc& c, cudaStream_t stream);
cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                           const CUtensorMap& vmap, const pa_cache_desc& c, cudaStream_t stream);
// The prefix pass of cascade decode (same kernel, cascade items, partial output).
cudaError_t launch_cascade_prefix(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                                  const CUtensorMap& vmap, const pa_cache_desc& c, cudaStream_t stream);

// Query heads packed into one 128-row prefill tile (the rest of its rows are tokens).
int32_t prefill_heads_per_tile(int32_t group);
// Launch `kernel` with programmatic stream serialization (it may overlap the
// tail of the previous kernel on the stream; see griddepcontrol in the kernels).
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                           Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Resident CTAs per SM for a kernel using `smem` dynamic shared memory, from
// the device's shared-memory and register limits (and `cap`).
int32_t ctas_per_sm(const void* kernel, int threads, size_t smem, int cap);

// Opt-in launch trace on stderr (environment PA_LOG_LAUNCH=1).
void log_launch(const char* kernel, int grid, int block, size_t smem, int per_sm);

// KV heads one decode CTA streams together (adjacent heads; only without GQA),
// and query heads per decode unit (heads per CTA x KV heads per CTA).
int32_t decode_kv_heads_per_cta(int32_t group, const pa_cache_desc& c);
// Query heads per unit of the CUDA-core kernel (the tensor-core kernel's unit is the whole group).
int32_t decode_heads_per_unit(int32_t group, const pa_cache_desc& c);
// Heads of one GQA group handled together by one decode CTA.
int32_t decode_heads_per_cta(int32_t group);
// Decode smem stage geometry, used by the launcher and the API's checks.
int32_t num_sms();

}  // namespace pa
