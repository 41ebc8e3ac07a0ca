// Grouped-query decode attention on the 5th-generation tensor cores (tcgen05).
//
// Same result as the CUDA-core decode kernel (decode.cu): for sequence s with
// L keys and the GH query heads that share KV head hk,
// o_h = softmax(q_h . K[0:L]^T * scale) . V[0:L], keys gathered through the
// block table (the page table of "vLLM核心架构：PagedAttention原理、KV
// Cache管理、连续批处理机制", §"一、PagedAttention：虚拟内存的灵感"). The work
// partition (units, segments, partial slots) is the one in decode_common.cuh,
// so the same merge kernel combines split units.
//
// Why tensor cores here: with GH query heads per KV head every key row feeds
// GH dot products and GH rows of P.V. On CUDA cores that is ~40 instructions
// per key row at GH = 4 and the kernel becomes issue-bound well below the HBM
// roofline. As matrix products the same work is a handful of MMAs per
// 128-token tile, which leaves the SM free to keep HBM busy.
//
// Design (B200, one CTA per SM, persistent over its block range):
//  * A tile is 128 consecutive tokens of one unit (128/bs KV blocks). Its
//    scores are computed transposed, S^T = K Q^T, with the tokens on the MMA's
//    M = 128 (one TMEM lane per token) and the head group on N = 16 (GH of the
//    16 columns used). The K tile is the A operand exactly as TMA lands it:
//    K-major, 128-byte swizzle, one box {64, 1, bs, 1} per block and half.
//  * Then O^T += V^T P^T: V is the A operand in MN-major form (the same smem
//    tile, read along the head dimension), P^T the B operand written by the
//    softmax threads as bf16. O^T lives in TMEM (lane = head-dim column).
//  * Warp 4 issues the TMA loads (Q^T once per segment, K and V per block)
//    into a ring of NST 64 KiB stages; blocks past the segment are loaded
//    with an out-of-range block index, so TMA fills them with zeros.
//  * Warp 5 (one thread) issues the MMAs, one tile ahead on S so that the
//    next tile's scores are ready when the softmax threads finish this one.
//  * Warps 0-3: thread t owns token t of the tile. The warp max of each head
//    is one integer reduction on order-preserving bits; one barrier-or per
//    tile tells whether any head's running max grew by more than 2^8. Only
//    then do the warps exchange their maxima and rescale l and the O^T
//    columns; otherwise P = 2^(s - m) with the old reference m stays below
//    2^8 and nothing is rescaled. l is kept per thread (per token slot) and
//    reduced once per segment.
//  * V rows at or beyond L inside the last block hold stale bits (possibly
//    NaN); the owning thread zeroes them before the P.V MMA.
#include <math_constants.h>

#include "decode_common.cuh"
#include "pa_common.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr float kRescaleLog2 = 8.f;

template <int BS, int GH, int NST>
struct DecTcCfg {
  static constexpr int D = 128;
  static constexpr int kTile = 128;             // tokens per tile (MMA M)
  static constexpr int kBlk = kTile / BS;       // KV blocks per tile
  static constexpr int kN = 16;                 // MMA N: head columns (GH used)
  static constexpr int kHalfB = kTile * 128;    // one 64-column half of a K or V tile
  static constexpr int kKB = 2 * kHalfB;        // K tile (D = 128)
  static constexpr int kStageB = 2 * kKB;       // K + V tile
  static constexpr int kQB = 2 * kN * 128;      // Q^T tile: 16 rows x 2 halves
  static constexpr int kPB = 2 * kN * 128;      // P^T tile: 16 rows x 128 tokens
  static constexpr int kQOff = NST * kStageB;
  static constexpr int kPOff = kQOff + 2 * kQB;
  static constexpr int kBarOff = kPOff + 2 * kPB;
  // full[NST], empty[NST], q_full[2], q_empty[2], s_full[2], p_full[2], pv_done[2], mma_done
  static constexpr int kNumBars = 2 * NST + 11;
  static constexpr int kRedOff = kBarOff + kNumBars * 8;   // [4 warps][16] tile maxima
  static constexpr int kRed2Off = kRedOff + 4 * 16 * 4;     // [4 warps][16] l sums
  static constexpr int kTmemOff = kRed2Off + 4 * 16 * 4;
  static constexpr int kScanOff = kTmemOff + 16;
  static constexpr int kSeqOff = kScanOff + 32 * 4;
  static constexpr uint32_t kTmemCols = 64;     // S^T x 2 (16 columns each) + O^T (16)
  static constexpr uint32_t kSCol = 0, kOCol = 32;
  static constexpr uint32_t kIdescS = tc::idesc_bf16_f32(128, kN, 0, 0);
  static constexpr uint32_t kIdescO = tc::idesc_bf16_f32(128, kN, 1, 0);
  static constexpr int kThreads = 192;
  static constexpr int kFailCol = 15;           // red / red2 column carrying a warp's failure flag
  static_assert(GH == 2 || GH == 4 || GH == 8, "head group of 2, 4 or 8");
  static_assert(kTile % BS == 0 && kBlk <= 32, "tile of whole blocks");
  static_assert(kStageB % 1024 == 0 && kQB % 1024 == 0 && kPB % 1024 == 0, "1024-byte operand alignment");
  static size_t smem_bytes(int num_seqs) { return 1024 + kSeqOff + 4ull * (num_seqs + 1); }
};

// Walks this CTA's tiles in order: segments of [beg, end), each cut into
// tiles of up to kBlk blocks. Every role of the CTA walks the same sequence.
template <int kBlk>
struct TileWalk {
  const int* prefix;
  const int32_t* skip_blocks;
  int num_seqs, HG, cta;
  int64_t beg, end, next_b;
  Segment g;
  int tb;         // first logical block of the current tile
  int seg;        // segment counter (from 0)
  bool valid;

  __device__ __forceinline__ void start(const int* p, const int32_t* skip, int S, int hg, int64_t b0, int64_t b1,
                                        int c) {
    prefix = p;
    skip_blocks = skip;
    num_seqs = S;
    HG = hg;
    beg = b0;
    end = b1;
    cta = c;
    next_b = b0;
    seg = -1;
    next_segment();
  }
  __device__ __forceinline__ void next_segment() {
    valid = next_b < end;
    if (!valid) return;
    locate_segment(next_b, prefix, num_seqs, HG, beg, end, cta, g);
    apply_skip(skip_blocks, HG, cta, g);
    next_b += g.bhi - g.blo;
    tb = g.blo;
    ++seg;
  }
  __device__ __forceinline__ void next() {
    tb += kBlk;
    if (tb >= g.bhi) next_segment();
  }
  __device__ __forceinline__ bool first() const { return tb == g.blo; }
  __device__ __forceinline__ bool last() const { return tb + kBlk >= g.bhi; }
  __device__ __forceinline__ int blocks() const { return min(kBlk, g.bhi - tb); }
};

template <int BS, int GH, int NST>
__global__ void __launch_bounds__(192, 1)
    paged_decode_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap, const DecodeArgs a) {
  using C = DecTcCfg<BS, GH, NST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + NST;
  uint64_t* q_full = empty + NST;
  uint64_t* q_empty = q_full + 2;
  uint64_t* s_full = q_empty + 2;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* mma_done = pv_done + 2;
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);
  float* red2 = reinterpret_cast<float*>(smem + C::kRed2Off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemOff);
  int* warp_tot = reinterpret_cast<int*>(smem + C::kScanOff);
  int* prefix = reinterpret_cast<int*>(smem + C::kSeqOff);  // [S+1] decode blocks before seq s

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int HG = a.num_q_heads / GH;  // units per sequence (= KV heads)

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, C::kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  // Chained launch: only the set-up above overlaps the previous grid. Every
  // input (index arrays, q, the cache) may have been written by the kernel
  // just before this one on the stream, and its writes are guaranteed
  // visible only after this wait.
  grid_dependency_wait();

  // ---- decode blocks of every sequence, and their prefix
  int carry = 0;
  if (tid == 0) prefix[0] = 0;
  for (int base = 0; base < a.num_seqs; base += blockDim.x) {
    const int s = base + tid;
    int n = 0;
    if (s < a.num_seqs) {
      const int L = __ldg(a.context_lens + s);
      const int r0 = __ldg(a.query_start_loc + s);
      const int ql = __ldg(a.query_start_loc + s + 1) - r0;
      if (ql == 1) {
        const int skip = a.skip_blocks ? __ldg(a.skip_blocks + s) : 0;
        if (L < 1 || L > a.max_context_len || L > a.max_blocks_per_seq * BS || skip < 0 ||
            skip > (L + BS - 1) / BS) {
          raise_flag(a.status, PA_FLAG_CONTEXT_RANGE);
        } else {
          n = (L + BS - 1) / BS - skip;
        }
      }
    }
    int total;
    const int incl = block_inclusive_scan(n, warp_tot, total);
    if (s < a.num_seqs) prefix[s + 1] = carry + incl;
    carry += total;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // The grids chained after this one may start now: every input they read
  // was complete before this grid passed its wait, and each of them waits
  // for its own predecessor at most.
  launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const int64_t B = static_cast<int64_t>(prefix[a.num_seqs]) * HG;  // blocks of all units
  if (blockIdx.x == 0 && a.seq_prefix)
    for (int i = tid; i <= a.num_seqs; i += blockDim.x) a.seq_prefix[i] = prefix[i];
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * B / a.grid;
  const int64_t end = static_cast<int64_t>(blockIdx.x + 1) * B / a.grid;

  TileWalk<C::kBlk> it;
  it.start(prefix, a.skip_blocks, a.num_seqs, HG, beg, end, static_cast<int>(blockIdx.x));

  if (warp == 4) {
    // ================= producer: Q^T per segment, K and V per block (TMA)
    bool ok = true;
    uint32_t i = 0;  // tiles issued
    int last_seg = -1;
    for (; it.valid && ok; it.next(), ++i) {
      const Segment& g = it.g;
      if (it.seg != last_seg) {  // first tile of a segment: the unit's query rows
        last_seg = it.seg;
        const uint32_t j = static_cast<uint32_t>(it.seg);
        if (lane == 0) {
          ok = mbar_wait(&q_empty[j & 1], ((j >> 1) & 1) ^ 1, a.status, a.wait_limit_ns);
          if (ok) {
            uint8_t* qs = smem + C::kQOff + (j & 1) * C::kQB;
            const int row = __ldg(a.query_start_loc + g.s);
            mbar_arrive_expect_tx(&q_full[j & 1], 2 * GH * 128);
            tma_load_3d(qs, &qmap, &q_full[j & 1], 0, g.hg * GH, row);
            tma_load_3d(qs + C::kN * 128, &qmap, &q_full[j & 1], 64, g.hg * GH, row);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
        if (!ok) break;
      }
      // lane b gathers block tb + b of the tile; lanes past the segment load
      // block index -1, an out-of-range box that TMA fills with zeros
      int phys = -1;
      if (lane < it.blocks()) {
        phys = __ldg(a.block_tables + static_cast<size_t>(g.s) * a.max_blocks_per_seq + g.skip + it.tb + lane);
        if (phys < 0 || phys >= a.num_blocks) {
          raise_flag(a.status, PA_FLAG_BLOCK_RANGE);
          phys = -1;
        }
      }
      const uint32_t st = i % NST;
      if (lane == 0) {
        ok = mbar_wait(&empty[st], ((i / NST) & 1) ^ 1, a.status, a.wait_limit_ns);
        if (ok) mbar_arrive_expect_tx(&full[st], C::kStageB);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
      if (!ok) break;
      if (lane < C::kBlk) {
        uint8_t* ks = smem + st * C::kStageB + lane * BS * 128;
        uint8_t* vs = ks + C::kKB;
        tma_load_4d(ks, &kmap, &full[st], 0, g.hg, 0, phys);
        tma_load_4d(ks + C::kHalfB, &kmap, &full[st], 64, g.hg, 0, phys);
        tma_load_4d(vs, &vmap, &full[st], 0, g.hg, 0, phys);
        tma_load_4d(vs + C::kHalfB, &vmap, &full[st], 64, g.hg, 0, phys);
      }
    }
    // Before the CTA exits no copy may still be landing in its shared memory:
    // wait (bounded) for the last use of every stage and Q buffer.
    if (lane == 0) {
      for (uint32_t k = i > NST ? i - NST : 0; k < i; ++k)
        if (!mbar_drain(&full[k % NST], (k / NST) & 1, a.status)) break;
      for (int j = last_seg - 1; j <= last_seg; ++j)
        if (j >= 0 && !mbar_drain(&q_full[j & 1], (j >> 1) & 1, a.status)) break;
    }
    __syncwarp();
  } else if (warp == 5) {
    // ================= MMA issue (one thread)
    // Two cursors over the same tiles: S^T of tile ns (once its K tile and,
    // for a segment's first tile, its Q^T have landed, and the softmax threads
    // are done with the S buffer it overwrites), and O^T += V^T P^T of tile np
    // (once its P^T is written). Whichever is ready is issued, so a stage is
    // released as soon as its P.V product is issued, never held back behind
    // the next tile's data.
    if (lane == 0 && it.valid) {
      TileWalk<C::kBlk> sw = it, pw = it;
      uint32_t ns = 0, np = 0;
      bool ok = true;
      uint64_t t0 = 0;
      uint32_t spins = 0;
      while (pw.valid && ok) {
        bool progressed = false;
        if (sw.valid && ns <= np + 1) {
          const uint32_t st = ns % NST, j = static_cast<uint32_t>(sw.seg);
          if ((!sw.first() || mbar_test_wait(&q_full[j & 1], (j >> 1) & 1)) &&
              mbar_test_wait(&full[st], (ns / NST) & 1)) {
            tc::fence_after_sync();
            const uint32_t k_addr = smem_u32(smem + st * C::kStageB);
            const uint32_t q_addr = smem_u32(smem + C::kQOff + (j & 1) * C::kQB);
#pragma unroll
            for (int kk = 0; kk < C::D / 16; ++kk) {
              const uint32_t ka = k_addr + (kk >> 2) * C::kHalfB + (kk & 3) * 32;
              const uint32_t qa = q_addr + (kk >> 2) * (C::kN * 128) + (kk & 3) * 32;
              tc::mma_bf16(tmem + C::kSCol + (ns & 1) * 16, tc::sw128_desc(ka, 16, 1024),
                           tc::sw128_desc(qa, 16, 1024), C::kIdescS, kk > 0);
            }
            tc::commit(&s_full[ns & 1]);
            if (sw.last()) tc::commit(&q_empty[j & 1]);
            sw.next();
            ++ns;
            progressed = true;
          }
        }
        if (np < ns && mbar_test_wait(&p_full[np & 1], (np >> 1) & 1)) {
          tc::fence_after_sync();
          const uint32_t st = np % NST;
          const uint32_t v_addr = smem_u32(smem + st * C::kStageB + C::kKB);
          const uint32_t p_addr = smem_u32(smem + C::kPOff + (np & 1) * C::kPB);
          const bool acc0 = !pw.first();
#pragma unroll
          for (int kk = 0; kk < C::kTile / 16; ++kk) {
            const uint32_t va = v_addr + kk * 16 * 128;
            const uint32_t pa_ = p_addr + (kk >> 2) * (C::kN * 128) + (kk & 3) * 32;
            tc::mma_bf16(tmem + C::kOCol, tc::sw128_desc(va, C::kHalfB, 1024), tc::sw128_desc(pa_, 16, 1024),
                         C::kIdescO, acc0 || kk > 0);
          }
          tc::commit(&pv_done[np & 1]);
          tc::commit(&empty[st]);
          pw.next();
          ++np;
          progressed = true;
        }
        if (progressed) {
          t0 = 0;
        } else if ((++spins & 1023u) == 0) {  // bounded: give up after the wait limit without progress
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) {
            t0 = now;
          } else if (now - t0 >= a.wait_limit_ns || flag_raised(a.status, PA_FLAG_WAIT_TIMEOUT)) {
            raise_flag(a.status, PA_FLAG_WAIT_TIMEOUT);
            ok = false;
          }
        }
      }
      // no MMA may be in flight when TMEM is released
      tc::commit(mma_done);
      mbar_drain(mma_done, 0, a.status);
    }
    __syncwarp();
  } else {
    // ================= warps 0-3: thread t owns token t of each tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m_used[GH], l_t[GH];
    int L = 0, lim = 0, row = 0;
    bool failed = false;
    for (uint32_t i = 0; it.valid; it.next(), ++i) {
      const Segment& g = it.g;
      const uint32_t b = i & 1;
      if (it.first()) {
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          m_used[h] = -CUDART_INF_F;
          l_t[h] = 0.f;
        }
        L = __ldg(a.context_lens + g.s);
        lim = min(L, (g.skip + g.bhi) * BS);  // tokens this CTA owns end here
        row = __ldg(a.query_start_loc + g.s);
      }
      const int tok = (g.skip + it.tb) * BS + tid;
      const bool valid = tok < lim;
      failed = failed || !mbar_wait(&s_full[b], (i >> 1) & 1, a.status, a.wait_limit_ns);
      failed = __any_sync(0xffffffffu, failed);
      float sv[GH];
      if (!failed) {
        tc::fence_after_sync();
        tc::ld_cols<GH>(t_lane + C::kSCol + b * 16, sv);
        tc::wait_ld();
      }
      bool bump = false;
      float wm[GH];
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        sv[h] = (valid && !failed) ? sv[h] * a.scale_log2 : -CUDART_INF_F;
        wm[h] = warp_max(sv[h]);
        bump = bump || wm[h] > m_used[h] + kRescaleLog2;
      }
      // A failed warp forces the exchange below, where every warp sees it.
      if (barrier_or(1, 128, bump || failed)) {
        if (lane == 0) {
#pragma unroll
          for (int h = 0; h < GH; ++h) red[warp * 16 + h] = wm[h];
          red[warp * 16 + C::kFailCol] = failed ? 1.f : 0.f;
        }
        barrier_sync(2, 128);
        bool any_fail = false;
        float alpha[GH];
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          const float tm = fmaxf(fmaxf(red[h], red[16 + h]), fmaxf(red[32 + h], red[48 + h]));
          alpha[h] = 1.f;
          if (tm > m_used[h] + kRescaleLog2) {
            alpha[h] = fast_exp2(m_used[h] - tm);
            m_used[h] = tm;
          }
          l_t[h] *= alpha[h];
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) any_fail = any_fail || red[w * 16 + C::kFailCol] != 0.f;
        if (any_fail) break;  // the same decision in every softmax thread
        if (!it.first()) {
          // O^T holds the P.V products up to tile i-1: wait for them, then rescale
          failed = !mbar_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, a.status, a.wait_limit_ns);
          failed = __any_sync(0xffffffffu, failed);
          if (!failed) {
            tc::fence_after_sync();
            float ov[GH];
            tc::ld_cols<GH>(t_lane + C::kOCol, ov);
            tc::wait_ld();
#pragma unroll
            for (int h = 0; h < GH; ++h) ov[h] *= alpha[h];
            tc::st_cols<GH>(t_lane + C::kOCol, ov);
            tc::wait_st();
          }
        }
      }
      float p[GH];
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        p[h] = fast_exp2(sv[h] - m_used[h]);  // 0 for masked tokens
        l_t[h] += p[h];
      }
      // P^T buffer b was last read by the P.V MMA of tile i-2
      if (i >= 2) {
        failed = failed || !mbar_wait(&pv_done[b], ((i - 2) >> 1) & 1, a.status, a.wait_limit_ns);
        failed = __any_sync(0xffffffffu, failed);
      }
      if (!failed) {
        uint8_t* pb = smem + C::kPOff + b * C::kPB + (tid >> 6) * (C::kN * 128) + (tid & 7) * 2;
        const int chunk = (tid & 63) >> 3;
#pragma unroll
        for (int h = 0; h < GH; ++h)
          *reinterpret_cast<__nv_bfloat16*>(pb + h * 128 + ((chunk ^ (h & 7)) << 4)) = __float2bfloat16_rn(p[h]);
        // a V row past L inside a loaded block holds stale bits: zero it
        if (tok >= L && tid < it.blocks() * BS) {
          const uint32_t st = i % NST;
          if (mbar_wait(&full[st], (i / NST) & 1, a.status, a.wait_limit_ns)) {
            uint8_t* vrow = smem + st * C::kStageB + C::kKB + tid * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              *reinterpret_cast<uint4*>(vrow + c * 16) = make_uint4(0u, 0u, 0u, 0u);
              *reinterpret_cast<uint4*>(vrow + C::kHalfB + c * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
          }
        }
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);

      if (it.last()) {
        // ---- segment epilogue: O^T / l to the output rows or this CTA's partial
        failed = failed || !mbar_wait(&pv_done[b], (i >> 1) & 1, a.status, a.wait_limit_ns);
        failed = __any_sync(0xffffffffu, failed);
        float ov[GH];
        if (!failed) {
          tc::fence_after_sync();
          tc::ld_cols<GH>(t_lane + C::kOCol, ov);
          tc::wait_ld();
        }
        float lw[GH];
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          lw[h] = l_t[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) lw[h] += __shfl_xor_sync(0xffffffffu, lw[h], off);
        }
        if (lane == 0) {
#pragma unroll
          for (int h = 0; h < GH; ++h) red2[warp * 16 + h] = lw[h];
          red2[warp * 16 + C::kFailCol] = failed ? 1.f : 0.f;
        }
        barrier_sync(2, 128);
        bool any_fail = false;
#pragma unroll
        for (int w = 0; w < 4; ++w) any_fail = any_fail || red2[w * 16 + C::kFailCol] != 0.f;
        if (any_fail) break;
        const int d = tid;  // TMEM lane of O^T = head-dim column
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          const float l = (red2[h] + red2[16 + h]) + (red2[32 + h] + red2[48 + h]);
          const float o = ov[h] / l;
          if (g.slot < 0) {
            static_cast<__nv_bfloat16*>(a.out)[(static_cast<size_t>(row) * a.num_q_heads + g.hg * GH + h) * C::D + d] =
                __float2bfloat16_rn(o);
          } else {
            const size_t part = static_cast<size_t>(g.slot) * GH + h;
            a.part_o[part * C::D + d] = o;
            if (d == 0) a.part_lse[part] = m_used[h] + log2f(l);
          }
        }
        // red2 is rewritten at the next segment end; O^T by its first P.V MMA,
        // which waits for this thread's next p_full arrival (after this read).
        tc::fence_before_sync();
        barrier_sync(2, 128);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BS, int GH, int NST>
cudaError_t launch_tc_t(DecodeArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                        cudaStream_t stream) {
  using C = DecTcCfg<BS, GH, NST>;
  auto kern = paged_decode_tc_kernel<BS, GH, NST>;
  const size_t smem = C::smem_bytes(a.num_seqs);
  static int configured_smem[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && configured_smem[dev] < static_cast<int>(smem)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) {
      (void)cudaGetLastError();  // reported through the return value; do not leave it pending
      return e;
    }
    configured_smem[dev] = static_cast<int>(smem);
  }
  int grid = num_sms();  // one CTA per SM: the stage ring takes most of shared memory
  if (grid > decode_max_grid()) grid = decode_max_grid();
  if (const char* env = getenv("PA_DECODE_GRID")) {  // testing / tuning: cap the grid
    const int v = atoi(env);
    if (v >= 1 && v < grid) grid = v;
  }
  a.grid = grid;
  a.hpu = GH;
  log_launch("paged_decode_tc_kernel", grid, C::kThreads, smem, 1);
  return launch_chained(kern, dim3(grid), dim3(C::kThreads), smem, stream, qmap, kmap, vmap, a);
}

template <int BS, int GH>
cudaError_t launch_tc_nst(DecodeArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          cudaStream_t stream) {
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  // three 64 KiB stages when the per-sequence table leaves room, else two
  if (DecTcCfg<BS, GH, 3>::smem_bytes(a.num_seqs) <= static_cast<size_t>(optin))
    return launch_tc_t<BS, GH, 3>(a, qmap, kmap, vmap, stream);
  return launch_tc_t<BS, GH, 2>(a, qmap, kmap, vmap, stream);
}

template <int BS>
cudaError_t launch_tc_gh(DecodeArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                         cudaStream_t stream) {
  switch (a.num_q_heads / a.num_kv_heads) {
    case 2: return launch_tc_nst<BS, 2>(a, qmap, kmap, vmap, stream);
    case 4: return launch_tc_nst<BS, 4>(a, qmap, kmap, vmap, stream);
    default: return launch_tc_nst<BS, 8>(a, qmap, kmap, vmap, stream);
  }
}

}  // namespace

bool decode_tc_supported(int32_t group, const pa_cache_desc& c) {
  return c.dtype == PA_BF16 && c.head_dim == 128 && (group == 2 || group == 4 || group == 8);
}

bool decode_uses_tc(int32_t group, const pa_cache_desc& c, bool short_units) {
  (void)short_units;
  static const bool enabled = [] {
    const char* env = getenv("PA_DECODE_TC");
    return env && env[0] == '1';
  }();
  return enabled && decode_tc_supported(group, c);
}

cudaError_t launch_decode_tc(DecodeArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, const pa_cache_desc& c, cudaStream_t stream) {
  switch (c.block_size) {
    case 8: return launch_tc_gh<8>(a, qmap, kmap, vmap, stream);
    case 16: return launch_tc_gh<16>(a, qmap, kmap, vmap, stream);
    default: return launch_tc_gh<32>(a, qmap, kmap, vmap, stream);
  }
}

}  // namespace pa
