// Prefix pass of cascade decode on the 5th-generation tensor cores (tcgen05).
//
// Requests that share a prompt point at the same pages ("vLLM核心架构：
// PagedAttention原理、KV Cache管理、连续批处理机制", §"二、KV Cache管理：从浪费到极致复用");
// here the shared pages are also read once: the decode rows of a group's
// members are stacked into 128-row tiles and attend every key of each
// 256-token chunk of the shared blocks (the prefill chunk of
// "深入剖析nano-vLLM推理引擎架构：PagedAttention内存管理实现", §"可落地配置参数"),
// leaving one partial (O / l, log2-sum-exp) per member, head and chunk for the
// decode merge.
//
// Design (B200, one CTA per work item, persistent over items):
//  * Work items are (group, chunk of shared blocks, tile of 128/GH members,
//    head group); a tile holds 128 query rows: 128/GH members x the GH query
//    heads of one GQA group, so each gathered K/V tile serves every head.
//  * Warp 4 (producer) loads the Q tile with one TMA per 64 head-dim columns
//    and, per 64-key tile, each K/V block of the tile with TMA (box
//    {64, 1, bs, 1}, 128-byte swizzle) into a 2-stage ring.
//  * Thread 0 issues S = Q K^T (M=128, N=64, K=16 steps) into TMEM, then
//    O += P V (M=128, N=head_dim) into TMEM; tcgen05.commit signals mbarriers.
//  * Warps 0-3 own one row each (TMEM lane = row): load S, mask, online
//    softmax in fp32 (exp2 with the scale folded into log2 e), write P as bf16
//    into the K slot it no longer needs (128-byte swizzled K-major layout).
//    O in TMEM is rescaled only when a row's running max grows by more than
//    2^8, so most tiles skip the TMEM round trip.
//  * V rows at or beyond the chunk's keys are zeroed before the PV MMA so stale
//    bits cannot reach the output.
#include <math_constants.h>

#include "pa_common.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int kBN = 64;            // keys per tile
constexpr float kRescaleLog2 = 8.f;

template <int D, int BS, int GH, int NST>
struct PrefillCfg {
  static constexpr int kTOK = 128 / GH;          // query tokens per tile
  static constexpr int kHalves = D / 64;         // 128-byte column groups
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKBytes = kBN * D * 2;
  static constexpr int kVBytes = kBN * D * 2;
  static constexpr int kPBytes = 128 * kBN * 2;
  static constexpr bool kPInK = kKBytes >= kPBytes;
  static constexpr int kStageBytes = kKBytes + kVBytes;
  static constexpr int kNST = NST;  // K/V stages in the ring
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = kQBytes;
  static constexpr int kPOff = kStageOff + kNST * kStageBytes;
  static constexpr int kBarOff = kPOff + (kPInK ? 0 : kPBytes);
  static constexpr int kTmemOff = kBarOff + ((5 + 2 * NST) * 8 + 15) / 16 * 16;
  static constexpr int kScanOff = kTmemOff + 16;
  static constexpr int kSeqOff = kScanOff + 32 * 4;
  // S of two tiles (tile j+1's scores are computed during tile j's softmax), then O
  static constexpr uint32_t kTmemCols = (2 * kBN + D) <= 128 ? 128 : 256;
  static constexpr int kBlocksPerTile = kBN / BS;
  static constexpr uint32_t kIdescS = tc::idesc_bf16_f32(128, kBN, 0, 0);
  static constexpr uint32_t kIdescO = tc::idesc_bf16_f32(128, D, 0, 1);
  static size_t smem_bytes(int num_seqs) { return 1024 + kSeqOff + 12ull * (num_seqs + 1); }
};

__device__ __forceinline__ int prefill_scan(int x, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, off);
      if (lane >= off) t += y;
    }
    if (lane < nw) warp_tot[lane] = t;
  }
  __syncthreads();
  total = warp_tot[nw - 1];
  const int r = x + (warp > 0 ? warp_tot[warp - 1] : 0);
  __syncthreads();
  return r;
}

struct Item {
  int s, r0, q_len, L, t0, hq0, hk, ntile;
  int kb0, chunk;  // cascade prefix pass: first key block of the item's chunk, and its index
};

template <int D, int BS, int GH, bool CASC, int NST>
__global__ void __launch_bounds__(160, 2)
    cascade_prefix_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const PrefillArgs a) {
  using C = PrefillCfg<D, BS, GH, NST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem + C::kQOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* s_done = bars + 2;    // [2]: S of even / odd tiles
  uint64_t* o_done = bars + 4;
  uint64_t* kv_full = bars + 5;   // [NST]
  uint64_t* kv_empty = kv_full + NST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemOff);
  int* warp_tot = reinterpret_cast<int*>(smem + C::kScanOff);
  int* prefix = reinterpret_cast<int*>(smem + C::kSeqOff);
  int* clen = prefix + (a.num_seqs + 1);
  int* qrow = clen + a.num_seqs;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.num_q_heads / a.num_kv_heads;
  const int HGp = a.num_q_heads / GH;  // head groups per tile row set

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(&s_done[0], 1);
    mbar_init(&s_done[1], 1);
    mbar_init(o_done, 1);
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

  // ---- tiles of every prefill sequence
  int carry = 0;
  if (tid == 0) prefix[0] = 0;
  // Items: (sequence, 128-row tile, head group) over the prefill rows; in the
  // cascade prefix pass (group, chunk of shared blocks, member tile, head group)
  const int n_src = CASC ? a.num_groups : a.num_seqs;
  for (int base = 0; base < n_src; base += blockDim.x) {
    const int s = base + tid;
    int n = 0;
    if (s < n_src && !CASC) {
      const int L = __ldg(a.context_lens + s);
      const int r0 = __ldg(a.query_start_loc + s);
      const int ql = __ldg(a.query_start_loc + s + 1) - r0;
      clen[s] = L;
      qrow[s] = r0;
      if (ql > 1) {
        if (L < ql || L > a.max_context_len || L > a.max_blocks_per_seq * BS || r0 < 0 ||
            r0 + ql > a.num_q_tokens) {
          raise_flag(a.status, PA_FLAG_CONTEXT_RANGE);
        } else {
          n = ((ql + C::kTOK - 1) / C::kTOK) * HGp;
        }
      }
    } else if (s < n_src) {
      // group s: members lead .. lead + m - 1 (one decode row each, rows r0 ..),
      // sharing the first nb blocks of the leader's table
      const int lead = __ldg(a.groups + 2 * s);
      const int m = __ldg(a.groups + 2 * s + 1);
      const int nb = m > 0 && lead >= 0 && lead + m <= a.num_seqs ? __ldg(a.skip_blocks + lead) : 0;
      const int r0 = nb > 0 ? __ldg(a.query_start_loc + lead) : 0;
      clen[s] = nb;
      qrow[s] = r0;
      if (m > 0) {
        if (nb < 1 || lead < 0 || lead + m > a.num_seqs || nb * BS > __ldg(a.context_lens + lead) || r0 < 0 ||
            r0 + m > a.num_q_tokens) {
          raise_flag(a.status, PA_FLAG_CONTEXT_RANGE);
        } else {
          n = ((nb + a.l1_chunk_blocks - 1) / a.l1_chunk_blocks) * ((m + C::kTOK - 1) / C::kTOK) * HGp;
        }
      }
    }
    int total;
    const int incl = prefill_scan(n, warp_tot, total);
    if (s < n_src) prefix[s + 1] = carry + incl;
    carry += total;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int W = prefix[n_src];

  auto item_of = [&](int w) {
    int lo = 0, hi = n_src;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= w) lo = mid; else hi = mid;
    }
    Item it;
    const int r = w - prefix[lo];
    const int mt0 = r / HGp;
    const int hg = r - mt0 * HGp;
    it.r0 = qrow[lo];
    it.hq0 = hg * GH;
    it.hk = it.hq0 / G;
    if (!CASC) {
      it.s = lo;
      it.L = clen[lo];
      it.q_len = 0;
      it.t0 = mt0 * C::kTOK;
      it.kb0 = 0;
      it.chunk = 0;
    } else {
      // mt0 = chunk * member_tiles + member tile
      const int lead = __ldg(a.groups + 2 * lo);
      const int m = __ldg(a.groups + 2 * lo + 1);
      const int mtiles = (m + C::kTOK - 1) / C::kTOK;
      it.s = lead;
      it.q_len = m;
      it.chunk = mt0 / mtiles;
      it.t0 = (mt0 - it.chunk * mtiles) * C::kTOK;
      it.kb0 = it.chunk * a.l1_chunk_blocks;
      it.L = min(a.l1_chunk_blocks, clen[lo] - it.kb0) * BS;  // keys of this chunk
    }
    return it;
  };
  auto finish_item = [&](Item& it) {
    if (CASC) {  // every member row sees every key of the chunk
      it.ntile = (it.L + kBN - 1) / kBN;
      return;
    }
    it.q_len = __ldg(a.query_start_loc + it.s + 1) - it.r0;
    const int t_last = min(it.t0 + C::kTOK, it.q_len) - 1;
    const int p_max = it.L - it.q_len + t_last;
    it.ntile = p_max / kBN + 1;
  };

  if (warp == 4) {
    // ================= producer
    if (lane == 0) {
      uint32_t it_no = 0, gj = 0;
      for (int w = blockIdx.x; w < W; w += gridDim.x, ++it_no) {
        Item it = item_of(w);
        finish_item(it);
        const int* row = a.block_tables + static_cast<size_t>(it.s) * a.max_blocks_per_seq;
        const int nblk_valid = (it.L + BS - 1) / BS;
        mbar_wait(q_empty, (it_no & 1) ^ 1, a.status);
        mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h)
          tma_load_3d(q_s + h * 128 * 128, &qmap, q_full, h * 64, it.hq0, it.r0 + it.t0);
        for (int j = 0; j < it.ntile; ++j, ++gj) {
          const uint32_t st = gj % NST;
          mbar_wait(&kv_empty[st], ((gj / NST) & 1) ^ 1, a.status);
          uint8_t* ks = smem + C::kStageOff + st * C::kStageBytes;
          uint8_t* vs = ks + C::kKBytes;
          mbar_arrive_expect_tx(&kv_full[st], C::kStageBytes);
#pragma unroll
          for (int b = 0; b < C::kBlocksPerTile; ++b) {
            const int lb = j * C::kBlocksPerTile + b;
            int phys = -1;
            if (lb < nblk_valid) {
              phys = __ldg(row + it.kb0 + lb);
              if (phys < 0 || phys >= a.num_blocks) {
                raise_flag(a.status, PA_FLAG_BLOCK_RANGE);
                phys = -1;
              }
            }
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h) {
              tma_load_4d(ks + h * kBN * 128 + b * BS * 128, &kmap, &kv_full[st], h * 64, it.hk, 0, phys);
              tma_load_4d(vs + h * kBN * 128 + b * BS * 128, &vmap, &kv_full[st], h * 64, it.hk, 0, phys);
            }
          }
        }
      }
    }
    return;
  }

  // ================= warps 0-3: one query row per thread (TMEM lane = row)
  const int r = tid;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t o_col = 2 * kBN;
  const uint32_t q_addr = smem_u32(q_s);
  uint32_t it_no = 0, gj = 0;
  // thread 0: S of global tile g = Q K(g)^T into S buffer g & 1, once K(g) has landed
  auto issue_s = [&](uint32_t g) {
    const uint32_t sg = g & 1, stg = g % NST;
    mbar_wait(&kv_full[stg], (g / NST) & 1, a.status);
    tc::fence_after_sync();
    const uint32_t k_addr = smem_u32(smem + C::kStageOff + stg * C::kStageBytes);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off_q = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
      const uint32_t off_k = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
      tc::mma_bf16(tmem + sg * kBN, tc::sw128_desc(q_addr + off_q, 16, 1024), tc::sw128_desc(k_addr + off_k, 16, 1024),
                   C::kIdescS, kk > 0);
    }
    tc::commit(&s_done[sg]);
  };
  for (int w = blockIdx.x; w < W; w += gridDim.x, ++it_no) {
    Item it = item_of(w);
    finish_item(it);
    const int tok = it.t0 + r / GH;
    // last key this row may see (the whole chunk in the cascade prefix pass)
    const int lim = CASC ? it.L - 1 : min(it.L - it.q_len + tok, it.L - 1);
    float m_used = -CUDART_INF_F, l = 0.f;
    mbar_wait(q_full, it_no & 1, a.status);
    if (tid == 0) issue_s(gj);
    __syncwarp();
    for (int j = 0; j < it.ntile; ++j, ++gj) {
      const uint32_t st = gj % NST, sb = gj & 1;  // K/V stage, S buffer
      uint8_t* ks = smem + C::kStageOff + st * C::kStageBytes;
      uint8_t* vs = ks + C::kKBytes;
      uint8_t* ps = C::kPInK ? ks : smem + C::kPOff;
      mbar_wait(&s_done[sb], (gj >> 1) & 1, a.status);
      tc::fence_after_sync();
      float sv[kBN];
      tc::ld32(t_lane + sb * kBN, sv);
      tc::ld32(t_lane + sb * kBN + 32, sv + 32);
      tc::wait_ld();
      // The next tile's S goes to the other buffer, whose last reader (this
      // tile's predecessor) finished before the previous P.V was issued.
      // Issue it now if its K is already in, so it overlaps this softmax.
      bool next_issued = false;
      if (tid == 0 && j + 1 < it.ntile && mbar_test_wait(&kv_full[(gj + 1) % NST], ((gj + 1) / NST) & 1)) {
        issue_s(gj + 1);
        next_issued = true;
      }
      __syncwarp();
      const int kbase = j * kBN;
      // With a positive scale the row max is taken on the raw scores and the
      // scale is folded into the exponent's FMA below; the causal mask is
      // applied only on tiles that reach past this row's last visible key.
      // (four independent max chains instead of one 64-long chain)
      float sc = a.scale_log2;
      float mq[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
      if (sc > 0.f && kbase + kBN - 1 <= lim) {
#pragma unroll
        for (int c = 0; c < kBN; ++c) mq[c & 3] = fmaxf(mq[c & 3], sv[c]);
      } else if (sc > 0.f) {
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          if (kbase + c > lim) sv[c] = -CUDART_INF_F;
          mq[c & 3] = fmaxf(mq[c & 3], sv[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          sv[c] = (kbase + c <= lim) ? sv[c] * sc : -CUDART_INF_F;
          mq[c & 3] = fmaxf(mq[c & 3], sv[c]);
        }
        sc = 1.f;  // already scaled
      }
      float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * sc;
      // Rescale only when the running max grows by more than 2^8; otherwise
      // keep the old reference so P stays below 2^8 and O needs no update.
      const float m_new = fmaxf(m_used, mx);
      float alpha = 1.f;
      const bool bump = m_new > m_used + kRescaleLog2;
      if (bump) {
        alpha = fast_exp2(m_used - m_new);
        m_used = m_new;
      }
      if (j > 0 && __any_sync(0xffffffffu, bump)) {
        mbar_wait(o_done, (gj - 1) & 1, a.status);  // O holds every P.V up to tile j-1
        tc::fence_after_sync();
#pragma unroll 1
        for (int q = 0; q < D / 32; ++q) {
          float ov[32];
          tc::ld32(t_lane + o_col + 32 * q, ov);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tc::st32(t_lane + o_col + 32 * q, ov);
        }
        tc::wait_st();
      }
      l *= alpha;
      uint8_t* prow = ps + r * 128;
      float lq[4] = {0.f, 0.f, 0.f, 0.f};  // four independent partial sums of this tile
#pragma unroll
      for (int c8 = 0; c8 < kBN / 8; ++c8) {
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float p0 = fast_exp2(fmaf(sv[c8 * 8 + 2 * i], sc, -m_used));
          const float p1 = fast_exp2(fmaf(sv[c8 * 8 + 2 * i + 1], sc, -m_used));
          lq[i] += p0 + p1;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      l += (lq[0] + lq[1]) + (lq[2] + lq[3]);
      // zero V rows at or beyond L (stale tail of the last block)
      const int vz0 = it.L - kbase;
      if (vz0 < kBN) {
        mbar_wait(&kv_full[st], (gj / NST) & 1, a.status);
        const int z0 = vz0 > 0 ? vz0 : 0;
        const int nchunks = (kBN - z0) * C::kHalves * 8;
        for (int i = tid; i < nchunks; i += 128) {
          const int h = i / ((kBN - z0) * 8);
          const int rem = i - h * (kBN - z0) * 8;
          const int row = z0 + rem / 8, c = rem & 7;
          *reinterpret_cast<uint4*>(vs + h * kBN * 128 + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t p_addr = smem_u32(ps), v_addr = smem_u32(vs);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          tc::mma_bf16(tmem + o_col, tc::sw128_desc(p_addr + kk * 32, 16, 1024),
                       tc::sw128_desc(v_addr + kk * 16 * 128, kBN * 128, 1024), C::kIdescO, j > 0 || kk > 0);
        tc::commit(o_done);
        tc::commit(&kv_empty[st]);
        if (j == it.ntile - 1) tc::commit(q_empty);
        if (!next_issued && j + 1 < it.ntile) issue_s(gj + 1);
      }
      __syncwarp();
    }
    // ---- epilogue: O / l -> bf16 rows of this sequence
    mbar_wait(o_done, (gj - 1) & 1, a.status);
    tc::fence_after_sync();
    const float inv_l = 1.f / l;
    const bool row_ok = tok < it.q_len;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) +
                          (static_cast<size_t>(it.r0 + tok) * a.num_q_heads + it.hq0 + r % GH) * D;
    // cascade prefix pass: partial (O / l, log2-sum-exp) of member it.s + tok, this chunk
    const size_t l1_slot =
        (static_cast<size_t>(it.s + tok) * a.num_q_heads + it.hq0 + r % GH) * a.l1_max_chunks + it.chunk;
    if (CASC && row_ok) a.l1_lse[l1_slot] = m_used + log2f(l);
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
      float ov[32];
      tc::ld32(t_lane + o_col + 32 * q, ov);
      tc::wait_ld();
      if (CASC && row_ok) {
        float* po = a.l1_o + l1_slot * D + 32 * q;
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4)
          *reinterpret_cast<float4*>(po + 4 * v4) = make_float4(ov[4 * v4] * inv_l, ov[4 * v4 + 1] * inv_l,
                                                                ov[4 * v4 + 2] * inv_l, ov[4 * v4 + 3] * inv_l);
      } else if (row_ok) {
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h2 =
                __floats2bfloat162_rn(ov[v4 * 8 + 2 * i] * inv_l, ov[v4 * 8 + 2 * i + 1] * inv_l);
            pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(orow + 32 * q + 8 * v4) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    tc::fence_before_sync();
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
  tc::fence_before_sync();
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (warp == 0) tc::tmem_dealloc(tmem, C::kTmemCols);
  if (tid == 0) grid_dependency_wait();  // finish no earlier than the previous grid
}

template <int D, int BS, int GH, bool CASC, int NST>
cudaError_t launch_prefill_t(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, cudaStream_t stream) {
  using C = PrefillCfg<D, BS, GH, NST>;
  auto kern = cascade_prefix_kernel<D, BS, GH, CASC, NST>;
  const size_t smem = C::smem_bytes(a.num_seqs);
  static int configured_smem[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && configured_smem[dev] < static_cast<int>(smem)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();  // reported through the return value; do not leave it pending
      return e;
    }
    configured_smem[dev] = static_cast<int>(smem);
  }
  // TMEM holds 512 columns per SM; each CTA allocates kTmemCols of them.
  const int per_sm = ctas_per_sm(reinterpret_cast<const void*>(kern), 160, smem, 512 / C::kTmemCols);
  // max_query_len bounds the rows of a sequence (prefill) or the members of a
  // group (cascade); in the cascade pass each group also has its chunks
  const int64_t rows = CASC ? static_cast<int64_t>(a.num_groups) * a.l1_max_chunks : a.num_seqs;
  const int64_t bound = rows * (a.num_q_heads / GH) * ((a.max_query_len + C::kTOK - 1) / C::kTOK);
  const int64_t slots = static_cast<int64_t>(num_sms()) * per_sm;
  const int grid = static_cast<int>(bound < slots ? (bound > 0 ? bound : 1) : slots);
  // Chained launch: the prefill rows do not read anything the decode grid
  // writes, so this grid may start as soon as SMs free up; each CTA waits for
  // the previous grid before it exits, which keeps stream order for whatever
  // is launched after pa_attention.
  log_launch("cascade_prefix_kernel", grid, 160, smem, per_sm);
  return launch_chained(kern, dim3(grid), dim3(160), smem, stream, qmap, kmap, vmap, a);
}

// K/V ring depth. Two 32 KiB stages keep the CTA at ~100 KB of shared memory,
// so two CTAs share an SM and overlap each other's softmax and MMA chains;
// five stages at one CTA per SM measured slower (82.6 vs 66.6 us on the
// mixed batch's prefill rows).
constexpr int kPrefillStages = 2;

template <int D, int BS, int GH, bool CASC>
cudaError_t launch_prefill_st(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, cudaStream_t stream) {
  return launch_prefill_t<D, BS, GH, CASC, kPrefillStages>(a, qmap, kmap, vmap, stream);
}

template <int D, int BS, bool CASC>
cudaError_t launch_prefill_gh(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, int gh, cudaStream_t stream) {
  switch (gh) {
    case 16: return launch_prefill_st<D, BS, 16, CASC>(a, qmap, kmap, vmap, stream);
    case 8: return launch_prefill_st<D, BS, 8, CASC>(a, qmap, kmap, vmap, stream);
    case 4: return launch_prefill_st<D, BS, 4, CASC>(a, qmap, kmap, vmap, stream);
    case 2: return launch_prefill_st<D, BS, 2, CASC>(a, qmap, kmap, vmap, stream);
    default: return launch_prefill_st<D, BS, 1, CASC>(a, qmap, kmap, vmap, stream);
  }
}

template <int D, bool CASC>
cudaError_t launch_prefill_bs(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, int bs, int gh, cudaStream_t stream) {
  switch (bs) {
    case 8: return launch_prefill_gh<D, 8, CASC>(a, qmap, kmap, vmap, gh, stream);
    case 16: return launch_prefill_gh<D, 16, CASC>(a, qmap, kmap, vmap, gh, stream);
    default: return launch_prefill_gh<D, 32, CASC>(a, qmap, kmap, vmap, gh, stream);
  }
}

}  // namespace

cudaError_t launch_cascade_prefix(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                                  const CUtensorMap& vmap, const pa_cache_desc& c, cudaStream_t stream) {
  if (c.dtype != PA_BF16) return cudaErrorNotSupported;
  const int gh = prefill_heads_per_tile(a.num_q_heads / a.num_kv_heads);
  if (c.head_dim == 64) return launch_prefill_bs<64, true>(a, qmap, kmap, vmap, c.block_size, gh, stream);
  return launch_prefill_bs<128, true>(a, qmap, kmap, vmap, c.block_size, gh, stream);
}

}  // namespace pa
