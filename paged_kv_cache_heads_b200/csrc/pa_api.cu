// C ABI of libpa: host-side validation, TMA tensor-map encoding, the device
// status word, and dispatch to the kernels. See include/pa.h for the contract
// of every entry point.
#include <algorithm>
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "pa.h"
#include "pa_internal.h"

namespace pa {
namespace {

thread_local std::string g_last_error;

pa_status fail(pa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

pa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// The status word: one per device, in this library's device memory image
// (a file-scope device variable, no allocation). Kernels get its address.
__device__ unsigned g_status_word;

constexpr int kMaxDevices = 64;

cudaError_t status_ptr(unsigned** out) {
  static unsigned* cache[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return e;
    cache[dev] = static_cast<unsigned*>(p);
  }
  *out = cache[dev];
  return cudaSuccess;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

cudaError_t get_encoder(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
    if (err == cudaSuccess && (q != cudaDriverEntryPointSuccess || !p)) err = cudaErrorSymbolNotFound;
    cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  *fn = cached;
  return err;
}

struct MapKey {
  const void* base;
  int rank;
  uint64_t dims[5];
  uint64_t strides[4];
  uint32_t box[5];
  int dtype;
  int swizzle;
  bool operator==(const MapKey& o) const { return memcmp(this, &o, sizeof(MapKey)) == 0; }
};

// Encode (or fetch from a small cache) a tiled tensor map.
pa_status tensor_map(CUtensorMap* out, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, int dtype, int swizzle) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = rank;
  for (int i = 0; i < rank; ++i) key.dims[i] = dims[i], key.box[i] = box[i];
  for (int i = 0; i + 1 < rank; ++i) key.strides[i] = strides_bytes[i];
  key.dtype = dtype;
  key.swizzle = swizzle;
  static std::mutex mu;
  static MapKey keys[16];
  static CUtensorMap maps[16];
  static int used = 0, next = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (keys[i] == key) {
        *out = maps[i];
        return PA_OK;
      }
  }
  EncodeTiledFn enc = nullptr;
  cudaError_t e = get_encoder(&enc);
  if (e != cudaSuccess) return cuda_fail(e, "cuTensorMapEncodeTiled entry point");
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) d[i] = dims[i], b[i] = box[i], es[i] = 1;
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  const CUtensorMapDataType dt =
      dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUtensorMapSwizzle sw = swizzle == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUtensorMap m;
  CUresult r = enc(&m, dt, rank, const_cast<void*>(base), d, s, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
  std::lock_guard<std::mutex> lock(mu);
  keys[next] = key;
  maps[next] = m;
  next = (next + 1) % 16;
  if (used < 16) ++used;
  *out = m;
  return PA_OK;
}

// Cache as a 4-D tensor {head_dim, num_kv_heads, block_size, num_blocks}; the
// box is {box_d, box_heads, block_size, 1}: one block of box_heads adjacent heads.
pa_status cache_map(CUtensorMap* out, const void* cache, const pa_cache_desc& c, uint32_t box_d,
                    int swizzle, uint32_t box_heads = 1) {
  const uint64_t eb = c.dtype == PA_BF16 ? 2 : 4;
  const uint64_t dims[4] = {uint64_t(c.head_dim), uint64_t(c.num_kv_heads), uint64_t(c.block_size),
                            uint64_t(c.num_blocks)};
  const uint64_t strides[3] = {c.head_dim * eb, uint64_t(c.num_kv_heads) * c.head_dim * eb,
                               uint64_t(c.block_size) * c.num_kv_heads * c.head_dim * eb};
  const uint32_t box[4] = {box_d, box_heads, uint32_t(c.block_size), 1};
  return tensor_map(out, cache, 4, dims, strides, box, c.dtype, swizzle);
}

// ---------------------------------------------------------------- validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

pa_status check_cache(const pa_cache_desc* c) {
  if (!c) return fail(PA_ERR_INVALID_ARG, "cache descriptor is NULL");
  if (c->dtype != PA_BF16 && c->dtype != PA_FP32)
    return fail(PA_ERR_UNSUPPORTED, "dtype %d unsupported (PA_FP32=0, PA_BF16=1)", c->dtype);
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d unsupported (64 or 128)", c->head_dim);
  if (c->block_size != 8 && c->block_size != 16 && c->block_size != 32)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d unsupported (8, 16 or 32)", c->block_size);
  if (c->num_kv_heads < 1 || c->num_blocks < 1)
    return fail(PA_ERR_INVALID_ARG, "num_kv_heads %d / num_blocks %d must be >= 1", c->num_kv_heads,
                c->num_blocks);
  if (c->num_kv_heads > 256) return fail(PA_ERR_UNSUPPORTED, "num_kv_heads %d > 256", c->num_kv_heads);
  const uint64_t eb = c->dtype == PA_BF16 ? 2 : 4;
  const uint64_t row_vecs = uint64_t(c->num_kv_heads) * c->head_dim * eb / 16;
  if (uint64_t(c->num_blocks) * c->block_size * row_vecs >= (1ull << 40))
    return fail(PA_ERR_UNSUPPORTED, "cache larger than 16 TiB");
  return PA_OK;
}

constexpr int32_t kMaxSeqs = 8192;

}  // namespace

void set_last_error(const char* msg) { g_last_error = msg; }

namespace {
std::atomic<uint64_t> g_wait_limit_ns{PA_WAIT_LIMIT_NS};
}  // namespace

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

int32_t ctas_per_sm(const void* kernel, int threads, size_t smem, int cap) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  int smem_sm = 0, reserved = 0, regs_sm = 0, max_threads = 0;
  cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&max_threads, cudaDevAttrMaxThreadsPerMultiProcessor, dev);
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return 1;
  const int warps = (threads + 31) / 32;
  const int regs_warp = ((fa.numRegs * 32 + 255) / 256) * 256;  // allocation unit: 256 per warp
  int n = cap;
  if (smem + fa.sharedSizeBytes > 0) {
    const int by_smem = smem_sm / static_cast<int>(smem + fa.sharedSizeBytes + reserved);
    if (by_smem < n) n = by_smem;
  }
  if (regs_warp > 0) {
    const int by_regs = regs_sm / (regs_warp * warps);
    if (by_regs < n) n = by_regs;
  }
  if (max_threads / threads < n) n = max_threads / threads;
  return n < 1 ? 1 : n;
}

void log_launch(const char* kernel, int grid, int block, size_t smem, int per_sm) {
  static const bool on = [] {
    const char* e = getenv("PA_LOG_LAUNCH");
    return e && e[0] == '1';
  }();
  if (on) fprintf(stderr, "[libpa] %s grid=%d block=%d smem=%zu ctas/sm=%d\n", kernel, grid, block, smem, per_sm);
}

int32_t num_sms() {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_last_error(void) { return g_last_error.c_str(); }

const char* pa_version(void) { return "libpa 0.1 (sm_100a)"; }

pa_status pa_store_kv(const void* k, const void* v, const int32_t* slot_mapping, int32_t num_tokens,
                      void* k_cache, void* v_cache, const pa_cache_desc* cache, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens %d < 0", num_tokens);
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache)
    return fail(PA_ERR_INVALID_ARG, "pa_store_kv: NULL pointer argument");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "pa_store_kv: k, v and caches must be 16-byte aligned");
  const uint64_t eb = cache->dtype == PA_BF16 ? 2 : 4;
  const uint64_t n16 = uint64_t(cache->num_kv_heads) * cache->head_dim * eb / 16;
  if (2ull * uint64_t(num_tokens) * n16 >= (1ull << 32) ||
      uint64_t(cache->num_blocks) * cache->block_size >= (1ull << 31))
    return fail(PA_ERR_UNSUPPORTED, "pa_store_kv: call too large; split it");
  unsigned* status = nullptr;
  cudaError_t e = status_ptr(&status);
  if (e != cudaSuccess) return cuda_fail(e, "status word");
  e = launch_store_kv(k, v, slot_mapping, num_tokens, k_cache, v_cache, *cache, status,
                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "store_kv launch");
  return PA_OK;
}

pa_status pa_copy_blocks(const int32_t* src_dst_pairs, int32_t num_pairs, void* k_cache,
                         void* v_cache, const pa_cache_desc* cache, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_pairs < 0) return fail(PA_ERR_INVALID_ARG, "num_pairs %d < 0", num_pairs);
  if (num_pairs == 0) return PA_OK;
  if (!src_dst_pairs || !k_cache || !v_cache)
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: NULL pointer argument");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: caches must be 16-byte aligned");
  unsigned* status = nullptr;
  cudaError_t e = status_ptr(&status);
  if (e != cudaSuccess) return cuda_fail(e, "status word");
  e = launch_copy_blocks(src_dst_pairs, num_pairs, k_cache, v_cache, *cache, status,
                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "copy_blocks launch");
  return PA_OK;
}

namespace {
// Encode the decode tensor maps and launch the decode grid (tensor-core kernel
// for grouped bf16 heads of 128, CUDA-core kernel otherwise). *e receives the
// launch status; the return value reports a tensor-map failure.
pa_status launch_decode_path(DecodeArgs& a, const void* q, const void* k_cache, const void* v_cache,
                             int32_t num_q_heads, int32_t num_q_tokens, const pa_cache_desc* cache,
                             bool short_units, cudaStream_t s, cudaError_t* e) {
  pa_status st;
  const int32_t group = num_q_heads / cache->num_kv_heads;
  // q as a 3-D tensor {head_dim, num_q_heads, num_q_tokens}
  const uint64_t qd[3] = {uint64_t(cache->head_dim), uint64_t(num_q_heads), uint64_t(num_q_tokens)};
  const uint64_t qs[2] = {uint64_t(cache->head_dim) * 2, uint64_t(num_q_heads) * cache->head_dim * 2};
  CUtensorMap kmap, vmap;
  if (decode_uses_tc(group, *cache, short_units)) {
    // tensor-core decode: 64-column (128-byte) swizzled boxes, Q^T per KV head
    CUtensorMap qmap;
    const uint32_t qbox[3] = {64, uint32_t(group), 1};
    if ((st = tensor_map(&qmap, q, 3, qd, qs, qbox, PA_BF16, 128)) != PA_OK) return st;
    if ((st = cache_map(&kmap, k_cache, *cache, 64, 128)) != PA_OK) return st;
    if ((st = cache_map(&vmap, v_cache, *cache, 64, 128)) != PA_OK) return st;
    *e = launch_decode_tc(a, qmap, kmap, vmap, *cache, s);
  } else {
    const uint32_t kh = decode_kv_heads_per_cta(group, *cache);
    if ((st = cache_map(&kmap, k_cache, *cache, cache->head_dim, 0, kh)) != PA_OK) return st;
    if ((st = cache_map(&vmap, v_cache, *cache, cache->head_dim, 0, kh)) != PA_OK) return st;
    *e = launch_decode(a, kmap, vmap, *cache, s);
  }
  return PA_OK;
}

// Workspace layout of one call: partial outputs, their log-sum-exp, and the
// per-sequence decode block prefix. False for arguments the size query cannot use.
struct WorkspaceLayout {
  size_t bytes = 0, lse_off = 0, prefix_off = 0;
  // prefill rows: partition, partial outputs and their log-sum-exp
  size_t pf_split_off = 0, pf_o_off = 0, pf_lse_off = 0;
  int32_t pf_grid = 0;
};
bool workspace_layout(int32_t num_seqs, int32_t num_q_heads, int32_t max_query_len, int32_t max_context_len,
                      const pa_cache_desc* cache, WorkspaceLayout* w) {
  if (!cache || check_cache(cache) != PA_OK || num_seqs < 0 || num_q_heads < 1 || max_query_len < 0 ||
      max_context_len < 0 || num_q_heads % cache->num_kv_heads)
    return false;
  *w = WorkspaceLayout();
  if (max_query_len < 1 || num_seqs == 0) return true;
  // partial slot u + c for unit u = (sequence, head group) and covering CTA c,
  // sized for whichever decode kernel the call may choose
  const int32_t group = num_q_heads / cache->num_kv_heads;
  size_t parts = 0;
  for (int32_t gh : {decode_heads_per_unit(group, *cache), decode_tc_supported(group, *cache) ? group : 0}) {
    if (gh < 1) continue;
    const size_t slots = size_t(num_seqs) * (num_q_heads / gh) + size_t(decode_max_grid());
    parts = std::max(parts, slots * gh);
  }
  w->lse_off = (parts * cache->head_dim * 4 + 255) & ~size_t(255);
  w->prefix_off = (w->lse_off + parts * 4 + 255) & ~size_t(255);
  w->bytes = w->prefix_off + (size_t(num_seqs) + 1) * 4;
  if (max_query_len > 1 && cache->dtype == PA_BF16) {
    // two partial slots of 256 rows per prefill CTA
    w->pf_grid = prefill_grid(num_seqs, num_q_heads, cache->num_kv_heads, max_query_len, max_context_len);
    const size_t rows = size_t(2) * w->pf_grid * 256;
    w->pf_split_off = (w->bytes + 255) & ~size_t(255);
    w->pf_o_off = (w->pf_split_off + size_t(w->pf_grid) * 16 + 255) & ~size_t(255);
    w->pf_lse_off = (w->pf_o_off + rows * cache->head_dim * 2 + 255) & ~size_t(255);  // fp16 O / l rows
    w->bytes = w->pf_lse_off + rows * 4;
  }
  return true;
}
}  // namespace

size_t pa_attention_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t max_query_len,
                                   int32_t max_context_len, const pa_cache_desc* cache) {
  WorkspaceLayout w;
  if (!workspace_layout(num_seqs, num_q_heads, max_query_len, max_context_len, cache, &w)) return 0;
  return w.bytes;
}

pa_status pa_attention(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                       const int32_t* context_lens, const int32_t* query_start_loc,
                       int32_t num_seqs, int32_t num_q_tokens, int32_t num_q_heads,
                       int32_t max_query_len, int32_t max_context_len, float scale,
                       const pa_cache_desc* cache, void* out, void* workspace,
                       size_t workspace_bytes, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_tokens < 0 || max_query_len < 0 || max_context_len < 0)
    return fail(PA_ERR_INVALID_ARG, "pa_attention: negative size argument");
  if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads %d must be a positive multiple of num_kv_heads %d",
                num_q_heads, cache->num_kv_heads);
  if (max_blocks_per_seq < 1) return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq must be >= 1");
  if (num_seqs == 0 || num_q_tokens == 0 || max_query_len == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start_loc || !out)
    return fail(PA_ERR_INVALID_ARG, "pa_attention: NULL pointer argument");
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "pa_attention: q, out and caches must be 16-byte aligned");
  if (num_seqs > kMaxSeqs) return fail(PA_ERR_UNSUPPORTED, "num_seqs %d > %d", num_seqs, kMaxSeqs);
  if (max_query_len > num_q_tokens)
    return fail(PA_ERR_INVALID_ARG, "max_query_len %d > num_q_tokens %d", max_query_len, num_q_tokens);
  if (int64_t(max_blocks_per_seq) * cache->block_size > (1ll << 30))
    return fail(PA_ERR_UNSUPPORTED, "max_blocks_per_seq too large");
  if (max_query_len > 1 && cache->dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "query rows with q_len > 1 need a bf16 cache");
  if (max_query_len > 1) {
    // the prefill grid numbers key tiles of (token pair, head group) items in int32
    const int64_t gh = prefill_heads_per_tile(num_q_heads / cache->num_kv_heads);
    const int64_t tiles = (int64_t(num_q_tokens) / 2 + 1) * (num_q_heads / gh) * ((int64_t(max_context_len) + 63) / 64);
    if (tiles >= (1ll << 31)) return fail(PA_ERR_UNSUPPORTED, "prefill batch too large; split it");
  }
  if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");

  WorkspaceLayout wl;
  workspace_layout(num_seqs, num_q_heads, max_query_len, max_context_len, cache, &wl);
  const size_t need = wl.bytes;
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(PA_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", need,
                workspace ? workspace_bytes : size_t(0));
  if (need > 0 && !aligned16(workspace))
    return fail(PA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");

  unsigned* status = nullptr;
  cudaError_t e = status_ptr(&status);
  if (e != cudaSuccess) return cuda_fail(e, "status word");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float scale_log2 = static_cast<float>(double(scale) * 1.4426950408889634);

  DecodeArgs a;
  a.q = q;
  a.out = out;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start_loc = query_start_loc;
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + wl.lse_off);
  a.seq_prefix = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + wl.prefix_off);
  a.status = status;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = cache->num_kv_heads;
  a.num_blocks = cache->num_blocks;
  a.max_context_len = max_context_len;
  a.grid = 0;
  a.hpu = 1;
  a.scale_log2 = scale_log2;
  a.wait_limit_ns = wait_limit_ns();
  a.skip_blocks = nullptr;
  a.l1_o = nullptr;
  a.l1_lse = nullptr;
  a.l1_max_chunks = 0;
  a.l1_chunk_blocks = 1;

  const int32_t group = num_q_heads / cache->num_kv_heads;
  const uint64_t qd[3] = {uint64_t(cache->head_dim), uint64_t(num_q_heads), uint64_t(num_q_tokens)};
  const uint64_t qs[2] = {uint64_t(cache->head_dim) * 2, uint64_t(num_q_heads) * cache->head_dim * 2};
  if ((st = launch_decode_path(a, q, k_cache, v_cache, num_q_heads, num_q_tokens, cache, false, s, &e)) != PA_OK)
    return st;
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  e = launch_decode_combine(a, *cache, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  if (max_query_len > 1) {
    PrefillArgs p;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.out = out;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start_loc = query_start_loc;
    p.status = status;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = cache->num_kv_heads;
    p.num_blocks = cache->num_blocks;
    p.max_context_len = max_context_len;
    p.max_query_len = max_query_len;
    p.num_q_tokens = num_q_tokens;
    p.scale_log2 = scale_log2;
    p.wait_limit_ns = wait_limit_ns();
    p.groups = nullptr;
    p.skip_blocks = nullptr;
    p.num_groups = 0;
    p.l1_o = nullptr;
    p.l1_lse = nullptr;
    p.l1_max_chunks = 0;
    p.l1_chunk_blocks = 1;
    p.pf_split = reinterpret_cast<int4*>(static_cast<char*>(workspace) + wl.pf_split_off);
    p.pf_o = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) + wl.pf_o_off);
    p.pf_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + wl.pf_lse_off);
    p.grid = wl.pf_grid;
    // K/V boxes are 64 columns wide (128 bytes) to match the 128-byte swizzle
    // of the MMA tiles.
    const int32_t gh = prefill_heads_per_tile(group);
    const uint32_t qbox[3] = {64, uint32_t(gh), uint32_t(128 / gh)};
    CUtensorMap qmap, pk, pv;
    if ((st = tensor_map(&qmap, q, 3, qd, qs, qbox, PA_BF16, 128)) != PA_OK) return st;
    if ((st = cache_map(&pk, k_cache, *cache, 64, 128)) != PA_OK) return st;
    if ((st = cache_map(&pv, v_cache, *cache, 64, 128)) != PA_OK) return st;
    e = launch_prefill(p, qmap, pk, pv, *cache, s);
    if (e == cudaErrorNotSupported) return fail(PA_ERR_UNSUPPORTED, "prefill rows not supported yet");
    if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  }
  return PA_OK;
}

}  // extern "C"

namespace {
// Cascade decode: the prefix pass splits each group's shared blocks into
// chunks of this many tokens (one work item per chunk and member tile).
constexpr int32_t kCascadeChunkTokens = 256;
int32_t cascade_chunk_blocks(const pa_cache_desc& c) { return kCascadeChunkTokens / c.block_size; }
int32_t cascade_max_chunks(int32_t max_shared_blocks, const pa_cache_desc& c) {
  return ceil_div(max_shared_blocks, cascade_chunk_blocks(c));
}
struct CascadeLayout {
  WorkspaceLayout base;
  size_t l1_o_off = 0, l1_lse_off = 0, bytes = 0;
};
bool cascade_layout(int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len, int32_t max_shared_blocks,
                    const pa_cache_desc* cache, CascadeLayout* w) {
  if (!workspace_layout(num_seqs, num_q_heads, 1, max_context_len, cache, &w->base) || max_shared_blocks < 0)
    return false;
  if (num_seqs == 0) return true;
  const size_t rows = size_t(num_seqs) * num_q_heads * size_t(cascade_max_chunks(max_shared_blocks, *cache));
  w->l1_o_off = (w->base.bytes + 255) & ~size_t(255);
  w->l1_lse_off = (w->l1_o_off + rows * cache->head_dim * 4 + 255) & ~size_t(255);
  w->bytes = w->l1_lse_off + rows * 4;
  return true;
}
}  // namespace

extern "C" {

size_t pa_attention_cascade_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len,
                                           int32_t max_shared_blocks, const pa_cache_desc* cache) {
  CascadeLayout w;
  if (!cascade_layout(num_seqs, num_q_heads, max_context_len, max_shared_blocks, cache, &w)) return 0;
  return w.bytes;
}

pa_status pa_attention_cascade(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* context_lens, const int32_t* query_start_loc, int32_t num_seqs,
                               int32_t num_q_heads, int32_t max_context_len, const int32_t* shared_blocks,
                               const int32_t* groups, int32_t num_groups, int32_t max_group_size,
                               int32_t max_shared_blocks, float scale, const pa_cache_desc* cache, void* out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || max_context_len < 0 || num_groups < 0 || max_group_size < 0 || max_shared_blocks < 0)
    return fail(PA_ERR_INVALID_ARG, "pa_attention_cascade: negative size argument");
  if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads %d must be a positive multiple of num_kv_heads %d",
                num_q_heads, cache->num_kv_heads);
  if (max_blocks_per_seq < 1) return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq must be >= 1");
  if (num_seqs == 0) return PA_OK;
  if (cache->dtype != PA_BF16) return fail(PA_ERR_UNSUPPORTED, "cascade decode needs a bf16 cache");
  if (num_groups > num_seqs) return fail(PA_ERR_INVALID_ARG, "more groups than sequences");
  if (num_groups > 0 && (!shared_blocks || !groups || max_group_size < 1 || max_shared_blocks < 1))
    return fail(PA_ERR_INVALID_ARG, "groups need shared_blocks, groups and positive bounds");
  if (max_shared_blocks > max_blocks_per_seq)
    return fail(PA_ERR_INVALID_ARG, "max_shared_blocks %d > max_blocks_per_seq %d", max_shared_blocks,
                max_blocks_per_seq);
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start_loc || !out)
    return fail(PA_ERR_INVALID_ARG, "pa_attention_cascade: NULL pointer argument");
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "pa_attention_cascade: q, out and caches must be 16-byte aligned");
  if (num_seqs > kMaxSeqs) return fail(PA_ERR_UNSUPPORTED, "num_seqs %d > %d", num_seqs, kMaxSeqs);
  if (int64_t(max_blocks_per_seq) * cache->block_size > (1ll << 30))
    return fail(PA_ERR_UNSUPPORTED, "max_blocks_per_seq too large");
  if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");
  CascadeLayout wl;
  cascade_layout(num_seqs, num_q_heads, max_context_len, num_groups > 0 ? max_shared_blocks : 0, cache, &wl);
  if (!workspace || workspace_bytes < wl.bytes)
    return fail(PA_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", wl.bytes,
                workspace ? workspace_bytes : size_t(0));
  if (!aligned16(workspace)) return fail(PA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");

  unsigned* status = nullptr;
  cudaError_t e = status_ptr(&status);
  if (e != cudaSuccess) return cuda_fail(e, "status word");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float scale_log2 = static_cast<float>(double(scale) * 1.4426950408889634);
  char* ws = static_cast<char*>(workspace);
  const int32_t chunk_blocks = cascade_chunk_blocks(*cache);
  const int32_t max_chunks = num_groups > 0 ? cascade_max_chunks(max_shared_blocks, *cache) : 0;

  DecodeArgs a;
  a.q = q;
  a.out = out;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start_loc = query_start_loc;
  a.part_o = reinterpret_cast<float*>(ws);
  a.part_lse = reinterpret_cast<float*>(ws + wl.base.lse_off);
  a.seq_prefix = reinterpret_cast<int32_t*>(ws + wl.base.prefix_off);
  a.status = status;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = cache->num_kv_heads;
  a.num_blocks = cache->num_blocks;
  a.max_context_len = max_context_len;
  a.grid = 0;
  a.hpu = 1;
  a.scale_log2 = scale_log2;
  a.wait_limit_ns = wait_limit_ns();
  a.skip_blocks = num_groups > 0 ? shared_blocks : nullptr;
  a.l1_o = reinterpret_cast<float*>(ws + wl.l1_o_off);
  a.l1_lse = reinterpret_cast<float*>(ws + wl.l1_lse_off);
  a.l1_max_chunks = max_chunks;
  a.l1_chunk_blocks = chunk_blocks;

  // 1. every sequence's own blocks (past its group's shared ones): partials
  // the suffix pass: each sequence's own blocks are typically few
  if ((st = launch_decode_path(a, q, k_cache, v_cache, num_q_heads, num_seqs, cache, num_groups > 0, s, &e)) !=
      PA_OK)
    return st;
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  // 2. each group's shared blocks, read once for all its members: partials
  if (num_groups > 0) {
    PrefillArgs p;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.out = out;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start_loc = query_start_loc;
    p.status = status;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = cache->num_kv_heads;
    p.num_blocks = cache->num_blocks;
    p.max_context_len = max_context_len;
    p.max_query_len = max_group_size;
    p.num_q_tokens = num_seqs;
    p.scale_log2 = scale_log2;
    p.wait_limit_ns = wait_limit_ns();
    p.groups = groups;
    p.skip_blocks = shared_blocks;
    p.num_groups = num_groups;
    p.l1_o = reinterpret_cast<float*>(ws + wl.l1_o_off);
    p.l1_lse = reinterpret_cast<float*>(ws + wl.l1_lse_off);
    p.l1_max_chunks = max_chunks;
    p.l1_chunk_blocks = chunk_blocks;
    p.pf_split = nullptr;
    p.pf_o = nullptr;
    p.pf_lse = nullptr;
    p.grid = 0;
    const int32_t gh = prefill_heads_per_tile(num_q_heads / cache->num_kv_heads);
    const uint64_t qd[3] = {uint64_t(cache->head_dim), uint64_t(num_q_heads), uint64_t(num_seqs)};
    const uint64_t qs[2] = {uint64_t(cache->head_dim) * 2, uint64_t(num_q_heads) * cache->head_dim * 2};
    const uint32_t qbox[3] = {64, uint32_t(gh), uint32_t(128 / gh)};
    CUtensorMap qmap, pk, pv;
    if ((st = tensor_map(&qmap, q, 3, qd, qs, qbox, PA_BF16, 128)) != PA_OK) return st;
    if ((st = cache_map(&pk, k_cache, *cache, 64, 128)) != PA_OK) return st;
    if ((st = cache_map(&pv, v_cache, *cache, 64, 128)) != PA_OK) return st;
    e = launch_cascade_prefix(p, qmap, pk, pv, *cache, s);
    if (e != cudaSuccess) return cuda_fail(e, "cascade prefix launch");
  }
  // 3. merge: the prefix grid finishes no earlier than the decode grid
  e = launch_decode_combine(a, *cache, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  return PA_OK;
}

uint64_t pa_set_wait_limit_ns(uint64_t limit_ns) {
  return g_wait_limit_ns.exchange(limit_ns, std::memory_order_relaxed);
}

pa_status pa_get_debug_status(void* stream, int32_t* host_flag) {
  if (!host_flag) return fail(PA_ERR_INVALID_ARG, "host_flag is NULL");
  unsigned* word = nullptr;
  cudaError_t e = status_ptr(&word);
  if (e != cudaSuccess) return cuda_fail(e, "status word");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Read, then clear, in stream order; only this stream is waited for.
  unsigned v = 0;
  e = cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(word, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  *host_flag = static_cast<int32_t>(v);
  return PA_OK;
}

pa_status pa_read_device_flags(uint32_t* flags, int32_t clear) {
  if (!flags) return fail(PA_ERR_INVALID_ARG, "flags is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  *flags = v;
  if (clear) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clear status word");
  }
  return PA_OK;
}

}  // extern "C"
