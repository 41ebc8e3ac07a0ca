/*
 * pa.h -- C ABI of libpa, the paged KV-cache hot path for NVIDIA B200 (sm_100a).
 *
 * Pages this interface restates (titles as published):
 *   [A] "深入剖析nano-vLLM推理引擎架构：PagedAttention内存管理实现"
 *   [B] "深入解析 nano-vLLM 推理引擎的分页 KV 缓存与内存优化架构"
 *   [C] "vLLM核心架构：PagedAttention原理、KV Cache管理、连续批处理机制"
 *
 * Cache layout (all calls): K and V caches are separate, contiguous arrays
 *   [num_blocks, block_size, num_kv_heads, head_dim]
 * of the cache dtype. Slot s is row s of the flat view
 *   [num_blocks * block_size, num_kv_heads * head_dim]
 * ([B] §"分页 KV 缓存的核心机制" flattens the cache to slots; the heads axis is kept).
 *
 * Conventions shared by every call:
 *  - Ownership: the caller owns every buffer, host and device. The library
 *    never allocates device memory; the only library-owned object is the
 *    host-side block manager handle (pa_bm_create / pa_bm_destroy).
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *    default stream). Kernel calls are asynchronous and never synchronise the
 *    host, except pa_read_device_flags, which says so.
 *  - Errors: arguments are checked on the host before anything is launched; a
 *    failed check returns a non-zero pa_status and launches nothing.
 *    pa_last_error() gives a message for the calling thread's last failure.
 *  - Device-side index checks: index *contents* (slots, block ids, context
 *    lengths, copy pairs) live in device memory and cannot be checked before
 *    launch. Kernels range-check each index they use; an out-of-range index
 *    is skipped (no memory access) and a bit is set in the library's device
 *    status word (PA_FLAG_*), read with pa_get_debug_status (one stream) or
 *    pa_read_device_flags (whole device). No kernel traps.
 *  - All indices are int32. Block-table rows are padded with -1; a negative
 *    slot means a padding token.
 *  - Device state: the library looks up the device addresses of its own
 *    device variables (the status word, the static workspace) once per
 *    device and keeps them for the life of the process. Do not use the
 *    library across cudaDeviceReset() or any other teardown of a device's
 *    primary context: the kept addresses would no longer be mapped.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* null pointer, negative count, inconsistent sizes */
  PA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype, head_dim, block_size...) */
  PA_ERR_CUDA = 3,          /* a CUDA runtime / driver call failed; see pa_last_error */
  PA_ERR_OUT_OF_BLOCKS = 4, /* block manager: free list too short; state unchanged */
  PA_ERR_INDEX = 5          /* block manager: unknown sequence or bad position */
} pa_status;

typedef enum { PA_FP32 = 0, PA_BF16 = 1 } pa_dtype;

/* Geometry of one K or V cache (both caches share it). Supported:
 * dtype PA_BF16 or PA_FP32; head_dim 64 or 128; block_size 8, 16 or 32;
 * num_kv_heads >= 1; num_blocks >= 1. */
typedef struct {
  int32_t num_blocks;
  int32_t block_size;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t dtype; /* pa_dtype */
} pa_cache_desc;

/* Bits of the device status word (pa_read_device_flags). */
#define PA_FLAG_SLOT_RANGE 0x1u    /* pa_store_kv: slot >= num_blocks * block_size */
#define PA_FLAG_BLOCK_RANGE 0x2u   /* pa_attention: block id outside [0, num_blocks) */
#define PA_FLAG_CONTEXT_RANGE 0x4u /* pa_attention: context_len > max_context_len or
                                      max_blocks_per_seq * block_size, or q_len > context_len */
#define PA_FLAG_PAIR_RANGE 0x8u    /* pa_copy_blocks: src or dst outside [0, num_blocks) */
#define PA_FLAG_WAIT_TIMEOUT 0x10u /* a bounded device-side wait gave up */

/* ------------------------------------------------------------------ kernels */

/*
 * pa_store_kv -- slot-mapped KV write ([B] §"分页 KV 缓存的核心机制"; blocks are
 * filled as tokens arrive, [A] §"PagedAttention：操作系统的内存智慧").
 *   k, v          device, [num_tokens, num_kv_heads, head_dim], cache dtype, contiguous
 *   slot_mapping  device int32 [num_tokens]; token t goes to slot slot_mapping[t];
 *                 negative = skip. Two tokens of one call must not share a slot.
 *   k_cache, v_cache  device caches (layout above), written in place.
 * A bit copy: cache rows receive exactly the bits of k and v.
 * Slots >= num_blocks*block_size are skipped and raise PA_FLAG_SLOT_RANGE.
 * num_tokens == 0 is a no-op.
 */
pa_status pa_store_kv(const void* k, const void* v, const int32_t* slot_mapping, int32_t num_tokens,
                      void* k_cache, void* v_cache, const pa_cache_desc* cache, void* stream);

/*
 * pa_copy_blocks -- copy-on-write block copy ([C] §"二、KV Cache管理：从浪费到极致复用":
 * a shared page is copied only when a request writes it, as in fork).
 *   src_dst_pairs device int32 [num_pairs, 2]; for each pair, block dst of
 *                 both caches becomes a copy of block src.
 * No dst may repeat or also appear as a src within one call (the block manager
 * never produces that); pairs with src == dst are no-ops. Out-of-range ids are
 * skipped and raise PA_FLAG_PAIR_RANGE. num_pairs == 0 is a no-op.
 */
pa_status pa_copy_blocks(const int32_t* src_dst_pairs, int32_t num_pairs, void* k_cache,
                         void* v_cache, const pa_cache_desc* cache, void* stream);

/*
 * pa_attention_workspace_size -- bytes of device workspace pa_attention needs
 * for these sizes: per-split partial outputs of decode rows and a small block
 * prefix; it grows with num_seqs * num_q_heads plus the device's SM count, not
 * with context length. 0 when num_seqs or max_query_len is 0. Same arguments
 * as the matching pa_attention call. Returns 0 for invalid arguments too; the
 * matching pa_attention call then reports the error.
 */
size_t pa_attention_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t max_query_len,
                                   int32_t max_context_len, const pa_cache_desc* cache);

/*
 * pa_attention -- attention of every query row over its sequence's keys,
 * gathered through the block table ([A] §"PagedAttention：操作系统的内存智慧",
 * [C] §"一、PagedAttention：虚拟内存的灵感"; prefill rows and decode rows,
 * [B] §"工程落地：配置参数与监控指标").
 *   q                device [num_q_tokens, num_q_heads, head_dim], cache dtype
 *   k_cache, v_cache device caches (read only)
 *   block_tables     device int32 [num_seqs, max_blocks_per_seq], row s maps
 *                    logical block i of sequence s to a physical block
 *   context_lens     device int32 [num_seqs]; L_s counts every key of
 *                    sequence s, including the rows queried now (store first)
 *   query_start_loc  device int32 [num_seqs + 1]; sequence s owns query rows
 *                    query_start_loc[s] .. query_start_loc[s+1]-1
 *   max_query_len    host bound on q_len_s (1 => decode-only batch)
 *   max_context_len  host bound on L_s; rows of a sequence with a larger L_s
 *                    are left unwritten and raise PA_FLAG_CONTEXT_RANGE
 *   scale            softmax scale (usually 1/sqrt(head_dim))
 *   out              device [num_q_tokens, num_q_heads, head_dim], cache dtype
 *   workspace        device scratch of at least pa_attention_workspace_size()
 *                    bytes (may be NULL when that is 0); contents are
 *                    overwritten; not shared by concurrent calls.
 * Row j of sequence s sits at position p = L_s - q_len_s + j and attends keys
 * 0..p; query head h uses KV head h / (num_q_heads / num_kv_heads).
 * num_q_heads must be a multiple of num_kv_heads. Rows with q_len_s > 1 need a
 * bf16 cache (tcgen05 tensor-core path); fp32 supports decode rows only.
 * Sequences with q_len_s == 0 are skipped. Rows of `out` not owned by any
 * sequence are not written.
 */
pa_status pa_attention(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                       const int32_t* context_lens, const int32_t* query_start_loc,
                       int32_t num_seqs, int32_t num_q_tokens, int32_t num_q_heads,
                       int32_t max_query_len, int32_t max_context_len, float scale,
                       const pa_cache_desc* cache, void* out, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * pa_attention_static_workspace -- pa_attention for callers that cannot
 * allocate device memory. The pages have no counterpart to this call; it
 * exists for callers such as a serving process whose device memory is handed
 * out entirely by its own pool, a plug-in host that does not let a library use
 * the CUDA allocator, or a latency-critical loop that must avoid cudaMalloc /
 * cudaFree (they can synchronise the device).
 *   Arguments and results are those of pa_attention, without the workspace:
 *   the split-K scratch is a fixed array of PA_STATIC_WORKSPACE_BYTES inside
 *   this library's device image, held on every GPU that loads the library
 *   until the process exits. No call allocates or frees anything.
 *   Batches whose pa_attention_workspace_size() exceeds the array are
 *   rejected with PA_ERR_UNSUPPORTED (and a message naming both sizes).
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 *   All calls on a device share the one array: calls that overlap on the GPU
 *   (different streams, or different host threads) race on it and must be
 *   serialised by the caller. Stale contents left by an earlier call are
 *   never read, so nothing needs clearing between calls.
 */
#define PA_STATIC_WORKSPACE_BYTES (16u << 20) /* 16 MiB */
pa_status pa_attention_static_workspace(const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                                        const int32_t* context_lens, const int32_t* query_start_loc,
                                        int32_t num_seqs, int32_t num_q_tokens, int32_t num_q_heads,
                                        int32_t max_query_len, int32_t max_context_len, float scale,
                                        const pa_cache_desc* cache, void* out, void* stream);

/*
 * pa_attention_cascade -- decode attention that reads shared prefix blocks
 * once per group ("vLLM核心架构：PagedAttention原理、KV Cache管理、连续批处理机制",
 * §"二、KV Cache管理：从浪费到极致复用": requests with a common prefix point at
 * the same pages; here the shared pages are also read only once).
 *
 * Same result as pa_attention for a batch of decode rows (every sequence has
 * exactly one query row: query_start_loc[s] = s, q is [num_seqs, Hq, D]):
 * out[s, h] = softmax(q[s, h] . K_s[0:L_s]^T * scale) . V_s[0:L_s].
 * Group g is the groups[2g+1] >= 2 consecutive sequences starting at
 * groups[2g] (groups are disjoint); every member s of a group has shared_blocks[s] = n_g,
 * the same n_g >= 1 leading block-table entries as the group's first member,
 * all of them full (n_g * block_size <= L_s). shared_blocks[s] = 0 for a
 * sequence in no group. The n_g shared blocks are attended once for all
 * members (a tensor-core pass over their stacked query rows, in chunks of 256
 * tokens); each member streams only its own blocks past them; the two partial
 * results are merged with their log-sum-exp weights.
 *   shared_blocks  device [num_seqs] int32     groups  device [num_groups][2] int32 (first, count)
 *   max_group_size >= the largest group; max_shared_blocks >= every n_g
 *                  (<= max_blocks_per_seq); both bound the launch and the workspace
 *   workspace      >= pa_attention_cascade_workspace_size(...) bytes, 16-byte aligned
 * bf16 caches only (PA_ERR_UNSUPPORTED otherwise). Other arguments, errors and
 * device flags as pa_attention; a group that breaks the rules above raises
 * PA_FLAG_CONTEXT_RANGE and its members' rows are unspecified.
 */
size_t pa_attention_cascade_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len,
                                           int32_t max_shared_blocks, const pa_cache_desc* cache);
pa_status pa_attention_cascade(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* context_lens, const int32_t* query_start_loc, int32_t num_seqs,
                               int32_t num_q_heads, int32_t max_context_len, const int32_t* shared_blocks,
                               const int32_t* groups, int32_t num_groups, int32_t max_group_size,
                               int32_t max_shared_blocks, float scale, const pa_cache_desc* cache, void* out,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_get_debug_status -- stream-ordered read of the device status word of the
 * current device: waits for the work queued on `stream` so far (only that
 * stream), writes the OR of the PA_FLAG_* bits raised since the word was last
 * cleared to *host_flag (0: no index was out of range and no wait gave up),
 * then clears the word. Flags raised by kernels on other streams that have not
 * finished are not waited for; use pa_read_device_flags for a device-wide read.
 *   stream     cudaStream_t as void* (NULL = legacy default stream)
 *   host_flag  host out
 * The index checks it reports are always compiled in (there is no separate
 * debug build): each index is compared once where it is used.
 */
pa_status pa_get_debug_status(void* stream, int32_t* host_flag);

/*
 * pa_read_device_flags -- read (and optionally clear) the device status word
 * of the current device. Synchronises the device first (all streams).
 *   flags  host out: OR of PA_FLAG_* raised since the last clear
 *   clear  non-zero: reset the word to 0 after reading
 */
pa_status pa_read_device_flags(uint32_t* flags, int32_t clear);

/*
 * pa_set_wait_limit_ns -- bound, in nanoseconds, of every device-side wait of
 * the kernels launched from now on (a consumer waiting for a copy, a producer
 * waiting for a free stage, a softmax warp waiting for an MMA). A wait that
 * runs out raises PA_FLAG_WAIT_TIMEOUT and its kernel winds down: its results
 * are unspecified, but every copy and MMA the kernel issued is waited for
 * (with the default bound) before its CTA exits, and the device stays usable.
 * Default 2 s (2000000000); 0 gives up on any wait not already satisfied,
 * which only a test of the timeout path wants. Process-wide, all devices.
 * Returns the previous limit.
 */
uint64_t pa_set_wait_limit_ns(uint64_t limit_ns);

/* Message for the calling thread's last non-OK status ("" if none). */
const char* pa_last_error(void);

/* Library version string. */
const char* pa_version(void);

/* ------------------------------------------------------------ block manager */

/*
 * Host-side block manager: free list, per-sequence block tables, reference
 * counts and copy-on-write ([A] §"PagedAttention：操作系统的内存智慧": free list
 * and block table, a new block only when the current one is full; [A]
 * §"连续批处理与内存管理的协同": a finished request returns its blocks; [C]
 * §"二、KV Cache管理：从浪费到极致复用": shared prefix pages, reference counts,
 * copy-on-write). It only produces int32 index arrays in host memory; it never
 * touches the GPU. Allocation takes blocks from the front of the free list,
 * freed blocks go to its back. A failing call changes no state.
 * A handle is not thread-safe; distinct handles are independent.
 */
typedef struct pa_bm pa_bm;

/* initial_free_order: host int32 [num_blocks], a permutation of 0..num_blocks-1
 * giving the initial free-list order, or NULL for 0, 1, 2, ... */
pa_status pa_bm_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_free_order,
                       pa_bm** out);
void pa_bm_destroy(pa_bm* bm);

/* New sequence holding num_tokens tokens (ceil(num_tokens/block_size) blocks).
 * slots_out: host int32 [num_tokens] receiving the slot of each token, or NULL. */
pa_status pa_bm_add_seq(pa_bm* bm, int64_t seq_id, int32_t num_tokens, int32_t* slots_out);

/* child shares the blocks holding parent's first num_tokens tokens (refcount +1
 * each); num_tokens < 0 means all of parent's tokens. */
pa_status pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child, int32_t num_tokens);

/* Append n tokens. slots_out: host int32 [n] (or NULL). If the last block is
 * partly filled and shared, it is replaced by a fresh block and the pair
 * (old, new) is written to cow_pair_out (host int32 [2], may be NULL) with
 * *num_cow_out = 1 (else 0); the caller copies old -> new (pa_copy_blocks)
 * before storing the new rows. */
pa_status pa_bm_append_tokens(pa_bm* bm, int64_t seq_id, int32_t n, int32_t* slots_out,
                              int32_t* cow_pair_out, int32_t* num_cow_out);

/* Drop the sequence; each of its blocks loses one reference and goes back to
 * the free list when it reaches 0 (in logical order). */
pa_status pa_bm_free_seq(pa_bm* bm, int64_t seq_id);

/* Slots of positions [start, start+n) of a sequence. out: host int32 [n]. */
pa_status pa_bm_slot_mapping(const pa_bm* bm, int64_t seq_id, int32_t start, int32_t n,
                             int32_t* out);

/* Block table rows for n sequences: table_out host int32 [n, max_blocks]
 * padded with -1; ctx_lens_out host int32 [n] (may be NULL). Fails with
 * PA_ERR_INVALID_ARG if a sequence holds more than max_blocks blocks. */
pa_status pa_bm_block_table(const pa_bm* bm, const int64_t* seq_ids, int32_t n, int32_t max_blocks,
                            int32_t* table_out, int32_t* ctx_lens_out);

int32_t pa_bm_num_free(const pa_bm* bm);
int32_t pa_bm_num_blocks(const pa_bm* bm);
/* Reference count of a block, or -1 if out of range. */
int32_t pa_bm_refcount(const pa_bm* bm, int32_t block);
/* Tokens held by a sequence, or -1 if unknown. */
int32_t pa_bm_seq_len(const pa_bm* bm, int64_t seq_id);
/* Copy up to cap free-list entries (front first) to out; returns the count. */
int32_t pa_bm_free_list(const pa_bm* bm, int32_t* out, int32_t cap);

/*
 * Groups for pa_attention_cascade, from the block tables of seq_ids (host, n
 * sequences, in batch order). Consecutive sequences form a group while the
 * number of leading block-table entries they all share, counting only blocks
 * full in every member, stays >= min_shared_blocks (>= 1); a group needs two
 * members or more. Writes shared_out[n] (that count for members, 0 for the
 * rest), groups_out (room for n/2 (first, count) pairs) and *num_groups_out.
 * Errors: PA_ERR_INVALID_ARG (NULL, n < 0, min_shared_blocks < 1), PA_ERR_INDEX
 * (unknown sequence).
 */
pa_status pa_bm_cascade_groups(const pa_bm* bm, const int64_t* seq_ids, int32_t n, int32_t min_shared_blocks,
                               int32_t* shared_out, int32_t* groups_out, int32_t* num_groups_out);

/*
 * Compaction ([A] §"连续批处理与内存管理的协同": defragmentation remaps blocks so
 * the used memory becomes dense, at the price of moving data). Every held
 * block ends in the id range [0, H), H = number of held blocks: the held
 * blocks with id >= H, in ascending order, move to the free ids below H, in
 * ascending order. Every table entry and reference count moves with its
 * block; the free list becomes H, H+1, ..., num_blocks-1.
 *
 * Writes the moves as (src, dst) int32 pairs to pairs_out (host memory, room
 * for `cap` pairs) and their count to *num_pairs_out. The caller copies the
 * K/V data with pa_copy_blocks(pairs, n, ...) before any attention that
 * reads the new tables (sources and destinations are disjoint, so one call in
 * any order suffices); n is the migration cost in blocks.
 * Errors: PA_ERR_INVALID_ARG for NULL arguments or when cap < n, in which case
 * *num_pairs_out is still set to n and nothing changes.
 */
pa_status pa_bm_compact(pa_bm* bm, int32_t* pairs_out, int32_t cap, int32_t* num_pairs_out);

/*
 * Block-manager statistics: the monitoring figures of [A] §"监控与调优要点"
 * (block utilisation, target 70-85%; internal fragmentation, retune the block
 * size above 20%; allocation latency P99, keep it under 1 ms; mapping-table
 * memory, keep it under 1% of the KV cache) plus the saving from prefix
 * sharing ([C] §"二、KV Cache管理：从浪费到极致复用").
 */
typedef struct {
  int32_t num_blocks;             /* pool size */
  int32_t free_blocks;            /* on the free list */
  int32_t held_blocks;            /* refcount > 0 */
  int32_t num_seqs;               /* live sequences */
  int64_t logical_blocks;         /* table entries of all sequences (a shared block counts per holder) */
  int64_t tokens;                 /* sum of sequence lengths */
  int64_t used_slots;             /* slots of held blocks that hold a token (a shared slot counts once) */
  double block_utilisation;       /* held_blocks / num_blocks */
  double internal_fragmentation;  /* 1 - used_slots / (held_blocks * block_size) (0 if nothing held) */
  double sharing_saving;          /* 1 - held_blocks / logical_blocks (0 if nothing held) */
  double table_bytes;             /* 4 bytes (one int32 physical id) per table entry */
  double table_overhead;          /* table_bytes / (num_blocks * kv_bytes_per_block): share of the whole KV pool */
  double alloc_p50_us;            /* latency of block-allocating calls (add_seq, append_tokens) */
  double alloc_p99_us;            /*   over the last (up to) 4096 such calls */
  int64_t alloc_samples;
} pa_bm_stats;

/* Fill *out. kv_bytes_per_block: K+V bytes one physical block occupies across
 * all layers (for table_overhead); pass 0 to leave table_overhead 0. A slot
 * counts as used when some live sequence maps one of its tokens to it, so a
 * shared block's used slots are those of the holder that wrote furthest.
 * The latency window holds the last 4096 block-allocating calls; both
 * percentiles are 0 before the first. Errors: PA_ERR_INVALID_ARG for NULL. */
pa_status pa_bm_get_stats(const pa_bm* bm, double kv_bytes_per_block, pa_bm_stats* out);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
