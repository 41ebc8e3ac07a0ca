// Slot-mapped KV write and copy-on-write block copy.
//
// Both are pure data movement bounded by HBM bandwidth: every byte is read
// once and written once, in 16-byte vectors, with consecutive threads on
// consecutive vectors of one contiguous row so that reads and writes coalesce
// into full 128-byte lines.
//
// Store: token t's K row and V row (num_kv_heads * head_dim elements each)
// go to flat cache row slot_mapping[t]; the write path of the page
// "深入解析 nano-vLLM 推理引擎的分页 KV 缓存与内存优化架构", §"分页 KV 缓存的核心机制".
// Copy: block dst := block src for both caches, the copy-on-write step of
// "vLLM核心架构：PagedAttention原理、KV Cache管理、连续批处理机制",
// §"二、KV Cache管理：从浪费到极致复用".
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Vector index i in [0, 2*T*n16): first all K vectors, then all V vectors;
// within a tensor, token-major then 16-byte column.
__global__ void __launch_bounds__(kThreads) store_kv_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, const int32_t* __restrict__ slots,
    uint32_t num_tokens, uint32_t n16, uint32_t num_slots, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, unsigned* status) {
  // A chained attention grid may start its prologue now; it waits for this
  // grid's completion before it reads the cache.
  launch_dependents();
  // The host guarantees total < 2^32, so every index below total fits in 32
  // bits; the loop counter itself is 64-bit so that the last step past total
  // cannot wrap around to a small value.
  const uint32_t per_tensor = num_tokens * n16;
  const uint64_t total = 2ull * per_tensor;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t base = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < total;
       base += stride * kUnroll) {
    uint4 r[kUnroll];
    uint4* dst[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      dst[u] = nullptr;
      const uint64_t i64 = base + u * stride;
      if (i64 < total) {
        const uint32_t i = static_cast<uint32_t>(i64);
        const bool is_v = i >= per_tensor;
        const uint32_t j = is_v ? i - per_tensor : i;
        const uint32_t t = j / n16;
        const uint32_t c = j - t * n16;
        const int32_t s = __ldg(slots + t);
        if (s >= 0) {
          if (static_cast<uint32_t>(s) < num_slots) {
            r[u] = ld_stream((is_v ? v : k) + j);
            dst[u] = (is_v ? v_cache : k_cache) + static_cast<size_t>(s) * n16 + c;
          } else if (c == 0 && !is_v) {
            raise_flag(status, PA_FLAG_SLOT_RANGE);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (dst[u]) *dst[u] = r[u];
  }
}

// One CTA per (pair, tensor, chunk of the block). Each block is
// block_size * num_kv_heads * head_dim elements, a multiple of 16 bytes.
__global__ void __launch_bounds__(kThreads) copy_blocks_kernel(const int32_t* __restrict__ pairs,
                                                              uint32_t n16_block, uint32_t num_blocks,
                                                              uint4* __restrict__ k_cache,
                                                              uint4* __restrict__ v_cache,
                                                              uint32_t chunks, unsigned* status) {
  launch_dependents();
  const uint32_t pair = blockIdx.x;
  const uint32_t tensor = blockIdx.y / chunks;
  const uint32_t chunk = blockIdx.y - tensor * chunks;
  const int32_t src = __ldg(pairs + 2 * pair);
  const int32_t dst = __ldg(pairs + 2 * pair + 1);
  if (src < 0 || dst < 0 || static_cast<uint32_t>(src) >= num_blocks ||
      static_cast<uint32_t>(dst) >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) raise_flag(status, PA_FLAG_PAIR_RANGE);
    return;
  }
  if (src == dst) return;
  uint4* cache = tensor ? v_cache : k_cache;
  const uint4* s = cache + static_cast<size_t>(src) * n16_block;
  uint4* d = cache + static_cast<size_t>(dst) * n16_block;
  const uint32_t per_chunk = (n16_block + chunks - 1) / chunks;
  const uint32_t lo = chunk * per_chunk;
  const uint32_t hi = min(n16_block, lo + per_chunk);
  for (uint32_t base = lo + threadIdx.x; base < hi; base += kThreads * kUnroll) {
    uint4 r[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t i = base + u * kThreads;
      if (i < hi) r[u] = ld_stream(s + i);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t i = base + u * kThreads;
      if (i < hi) d[i] = r[u];
    }
  }
}

}  // namespace

cudaError_t launch_store_kv(const void* k, const void* v, const int32_t* slots, int32_t num_tokens,
                            void* k_cache, void* v_cache, const pa_cache_desc& c, unsigned* status,
                            cudaStream_t stream) {
  const int eb = c.dtype == PA_BF16 ? 2 : 4;
  const uint32_t n16 = static_cast<uint32_t>(c.num_kv_heads) * c.head_dim * eb / 16;
  const uint64_t total = 2ull * static_cast<uint64_t>(num_tokens) * n16;
  const uint64_t want = (total + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  const uint64_t cap = static_cast<uint64_t>(num_sms()) * 16;
  const unsigned grid = static_cast<unsigned>(want < cap ? (want ? want : 1) : cap);
  const uint32_t num_slots = static_cast<uint32_t>(c.num_blocks) * c.block_size;
  store_kv_kernel<<<grid, kThreads, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), slots, num_tokens, n16, num_slots,
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), status);
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(const int32_t* pairs, int32_t num_pairs, void* k_cache,
                               void* v_cache, const pa_cache_desc& c, unsigned* status,
                               cudaStream_t stream) {
  const int eb = c.dtype == PA_BF16 ? 2 : 4;
  const uint32_t n16_block =
      static_cast<uint32_t>(c.block_size) * c.num_kv_heads * c.head_dim * eb / 16;
  // About 16 KiB per CTA: enough bytes in flight without too few CTAs.
  uint32_t chunks = (n16_block + 1023) / 1024;
  if (chunks < 1) chunks = 1;
  dim3 grid(static_cast<unsigned>(num_pairs), 2 * chunks);
  copy_blocks_kernel<<<grid, kThreads, 0, stream>>>(pairs, n16_block, c.num_blocks,
                                                    static_cast<uint4*>(k_cache),
                                                    static_cast<uint4*>(v_cache), chunks, status);
  return cudaGetLastError();
}

}  // namespace pa
