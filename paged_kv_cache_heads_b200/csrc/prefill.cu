// Chunked-prefill attention on the 5th-generation tensor cores (tcgen05).
//
// Rows of sequences with q_len > 1: row j of sequence s sits at position
// p = L - q_len + j and attends keys 0..p (causal inside the chunk, full over
// the cached context), keys gathered through the block table. This is the
// prefill call that the page "深入解析 nano-vLLM 推理引擎的分页 KV 缓存与内存优化架构",
// §"工程落地：配置参数与监控指标" hands to a variable-length attention kernel,
// here on a paged cache with the 256-token prefill chunks of the page
// "深入剖析nano-vLLM推理引擎架构：PagedAttention内存管理实现", §"可落地配置参数".
//
// Design (B200, one persistent CTA per SM, warp-specialised):
//  * A Q tile is 128 query rows: 128/GH tokens x the GH query heads of one GQA
//    group, so each gathered K/V tile serves every head of the group. A work
//    item (pair) is two consecutive Q tiles of one sequence and head group:
//    both tiles multiply the same K/V tiles, which halves the shared-memory
//    traffic per MMA and gives the tensor pipe two independent chains.
//  * Keys come in tiles of 64. Every pair's key tiles are numbered
//    contiguously (sequence, head group, pair) and the grid splits the whole
//    range evenly (stream-K): CTA c takes tiles [c*T/G, (c+1)*T/G), so long
//    and short pairs balance. A pair one CTA covers entirely is written
//    straight to the output; otherwise each covering CTA leaves a partial
//    (O / l, m + log2 l) per row and prefill_combine_kernel merges them.
//  * Warp 9 (producer) loads both Q tiles per segment and, per key tile, each
//    KV block of the tile with TMA (box {64, 1, bs, 1}, 128-byte swizzle) into
//    a ring of K/V stages.
//  * Warp 8 (one thread) issues S_i = Q_i K^T (M=128, N=64) into the TMEM
//    columns of Q tile i as soon as its softmax warps have loaded the previous
//    S into registers, so the next scores are computed during the current
//    softmax; and O_i += P_i V with P_i read from tensor memory (M=128,
//    N=head_dim). No MMA waits for another MMA: the tensor pipe stays fed.
//    tcgen05.commit arrives on mbarriers; every wait is bounded.
//  * Warps 0-3 and 4-7 run the softmax of Q tile 0 and 1: one row per thread
//    (TMEM lane = row), fp32 online softmax with exp2 on the scale folded into
//    log2 e, P written as bf16 into one of two TMEM P buffers of the tile (the
//    MMA reads it there). O is rescaled in TMEM only when a row's running max
//    grows by more than 2^8.
//  * V rows at or beyond L inside the last key tile hold stale bits; the MMA
//    warp zeroes them before the P.V product, so they cannot reach the output.
#include <math_constants.h>

#include "decode_common.cuh"
#include "pa_common.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int kBN = 64;             // keys per tile
constexpr float kRescaleLog2 = 8.f;
constexpr int kMinTilesPerCta = 8;  // a CTA gets at least this many key tiles of work
constexpr int kThreads = 320;       // softmax warps 0-7, MMA warp 8, producer warp 9
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;

template <int D, int BS, int GH>
struct PrefillCfg {
  static constexpr int kTOK = 128 / GH;      // query tokens per Q tile
  static constexpr int kPairTok = 2 * kTOK;  // query tokens per work item
  static constexpr int kHalves = D / 64;     // 128-byte column groups
  static constexpr int kQTileB = 128 * D * 2;
  static constexpr int kKB = kBN * D * 2;    // one K (or V) tile
  static constexpr int kStageB = 2 * kKB;
  static constexpr int kNST = D == 128 ? 4 : 6;  // K/V stages
  static constexpr int kBlk = kBN / BS;          // KV blocks per key tile
  static constexpr int kStageOff = 2 * kQTileB;
  static constexpr int kBarOff = kStageOff + kNST * kStageB;
  // q_full, q_empty, mma_done, kv_full[NST], kv_empty[NST], s_full[2], s_free[2], p_full[4], pv_done[4]
  static constexpr int kNumBars = 3 + 2 * kNST + 12;
  static constexpr int kTmemOff = kBarOff + kNumBars * 8;
  static constexpr int kScanOff = (kTmemOff + 16 + 15) / 16 * 16;
  static constexpr int kSeqOff = kScanOff + 32 * 4;
  // TMEM columns: S of Q tile i at 64 i; its P buffers b at 128 + 64 i + 32 b
  // (64 bf16 keys packed two per column); O of Q tile i at 256 + i * D.
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kPCol = 128;
  static constexpr uint32_t kOCol = 256;
  static constexpr uint32_t kIdescS = tc::idesc_bf16_f32(128, kBN, 0, 0);
  static constexpr uint32_t kIdescO = tc::idesc_bf16_f32(128, D, 0, 1);
  static size_t smem_bytes(int num_seqs) { return 1024 + kSeqOff + 4ull * (num_seqs + 1); }
};

// Key tiles a pair (or its first Q tile) needs: through the last visible key
// of its last row, tok_end being one past that row's token.
__device__ __forceinline__ int tiles_through(int L, int ql, int tok_end) { return (L - ql + tok_end - 1) / kBN + 1; }

// The part of one pair that one CTA processes.
struct PSeg {
  int s, hg, pt;     // sequence, head group, pair of that sequence
  int L, ql, r0;     // keys, query rows and first query row of the sequence
  int j_lo, j_hi;    // key tiles [j_lo, j_hi) of the pair
  int nt, nt0;       // key tiles of the pair, of its first Q tile
  int slot;          // -1: this CTA covers the whole pair; else its partial slot
  bool t1;           // the second Q tile holds at least one row of the sequence
};

// The segment of CTA `cta` (tile range [beg, end)) that starts at global key
// tile b. prefix[s] = key tiles before sequence s (prefix[num_seqs] > b).
template <int GH>
__device__ __forceinline__ void locate(int64_t b, int64_t beg, int64_t end, int cta, const int* prefix,
                                       int num_seqs, int HGp, const PrefillArgs& a, PSeg& g) {
  constexpr int TOK = 128 / GH, PT = 2 * TOK;
  int lo = 0, hi = num_seqs;  // prefix[lo] <= b < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= b) lo = mid; else hi = mid;
  }
  g.s = lo;
  g.L = __ldg(a.context_lens + lo);
  g.r0 = __ldg(a.query_start_loc + lo);
  g.ql = __ldg(a.query_start_loc + lo + 1) - g.r0;
  const int tiles_hg = (prefix[lo + 1] - prefix[lo]) / HGp;
  int off = static_cast<int>(b - prefix[lo]);
  g.hg = off / tiles_hg;
  off -= g.hg * tiles_hg;
  int pt = 0, nt;
  for (;;) {
    nt = tiles_through(g.L, g.ql, min((pt + 1) * PT, g.ql));
    if (off < nt) break;
    off -= nt;
    ++pt;
  }
  g.pt = pt;
  g.nt = nt;
  g.nt0 = tiles_through(g.L, g.ql, min(pt * PT + TOK, g.ql));
  g.t1 = pt * PT + TOK < g.ql;
  g.j_lo = off;
  const int64_t room = end - b;
  g.j_hi = off + static_cast<int>(room < nt - off ? room : nt - off);
  g.slot = (off == 0 && g.j_hi == nt) ? -1 : 2 * cta + (b > beg ? 1 : 0);
}

template <int D, int BS, int GH>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const PrefillArgs a) {
  using C = PrefillCfg<D, BS, GH>;
  constexpr int NST = C::kNST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* mma_done = bars + 2;
  uint64_t* kv_full = bars + 3;     // [NST]
  uint64_t* kv_empty = kv_full + NST;
  uint64_t* s_full = kv_empty + NST;  // [Q tile]: S computed
  uint64_t* s_free = s_full + 2;      // [Q tile]: S loaded into registers by the softmax warps
  uint64_t* p_full = s_free + 2;      // [Q tile * 2 + P buffer]
  uint64_t* pv_done = p_full + 4;     // [Q tile * 2 + P buffer]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemOff);
  int* warp_tot = reinterpret_cast<int*>(smem + C::kScanOff);
  int* prefix = reinterpret_cast<int*>(smem + C::kSeqOff);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.num_seqs;
  const int G = a.num_q_heads / a.num_kv_heads;
  const int HGp = a.num_q_heads / GH;  // head groups

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(mma_done, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);  // one arrival per softmax warp of the Q tile
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    fence_barrier_init();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }

  // ---- key tiles of every prefill sequence, and their prefix. This grid is
  // chained after the decode merge; every input it reads was complete before
  // the decode grid passed its own wait, which happened before any grid
  // chained after it could start.
  int carry = 0;
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + tid;
    int n = 0;
    if (s < S) {
      const int L = __ldg(a.context_lens + s);
      const int r0 = __ldg(a.query_start_loc + s);
      const int ql = __ldg(a.query_start_loc + s + 1) - r0;
      if (ql > 1) {
        if (L < ql || L > a.max_context_len || L > a.max_blocks_per_seq * BS || r0 < 0 ||
            r0 + ql > a.num_q_tokens) {
          raise_flag(a.status, PA_FLAG_CONTEXT_RANGE);
        } else {
          for (int pt = 0; pt * C::kPairTok < ql; ++pt) n += tiles_through(L, ql, min((pt + 1) * C::kPairTok, ql));
          n *= HGp;
        }
      }
    }
    int total;
    const int incl = block_inclusive_scan(n, warp_tot, total);
    if (s < S) prefix[s + 1] = carry + incl;
    carry += total;
  }
  if (tid == 0) prefix[0] = 0;
  __syncthreads();
  const int T = prefix[S];
  const int Geff = T > 0 ? min(static_cast<int>(gridDim.x), (T + kMinTilesPerCta - 1) / kMinTilesPerCta) : 1;
  if (blockIdx.x == 0) {  // the partition, for the merge kernel
    for (int i = tid; i <= S; i += blockDim.x) a.pf_prefix[i] = prefix[i];
    if (tid == 0) {
      a.pf_prefix[S + 1] = Geff;
      a.pf_prefix[S + 2] = T;
    }
  }
  if (T == 0 || static_cast<int>(blockIdx.x) >= Geff) {
    if (tid == 0) grid_dependency_wait();  // finish no earlier than the previous grid
    return;
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, C::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * T / Geff;
  const int64_t end = static_cast<int64_t>(blockIdx.x + 1) * T / Geff;
  const int cta = static_cast<int>(blockIdx.x);

  if (warp == kLoadWarp) {
    // ================= producer: Q tiles per segment, K/V blocks per key tile
    bool ok = true;
    uint32_t kt = 0, nq = 0;  // key tiles and Q loads issued
    for (int64_t b = beg; b < end && ok;) {
      PSeg g;
      locate<GH>(b, beg, end, cta, prefix, S, HGp, a, g);
      b += g.j_hi - g.j_lo;
      const int hq0 = g.hg * GH, hk = hq0 / G;
      const int t0 = g.pt * C::kPairTok;
      if (lane == 0) {
        ok = mbar_wait(q_empty, (nq & 1) ^ 1, a.status, a.wait_limit_ns);
        if (ok) {
          mbar_arrive_expect_tx(q_full, 2 * C::kQTileB);
#pragma unroll
          for (int qi = 0; qi < 2; ++qi)
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h)
              tma_load_3d(smem + qi * C::kQTileB + h * 128 * 128, &qmap, q_full, h * 64, hq0,
                          g.r0 + t0 + qi * C::kTOK);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
      if (!ok) break;
      ++nq;
      const int* row = a.block_tables + static_cast<size_t>(g.s) * a.max_blocks_per_seq;
      const int nblk_valid = (g.L + BS - 1) / BS;
      for (int j = g.j_lo; j < g.j_hi; ++j, ++kt) {
        const uint32_t st = kt % NST;
        if (lane == 0) {
          ok = mbar_wait(&kv_empty[st], ((kt / NST) & 1) ^ 1, a.status, a.wait_limit_ns);
          if (ok) mbar_arrive_expect_tx(&kv_full[st], C::kStageB);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
        if (!ok) break;
        if (lane < C::kBlk) {
          const int lb = j * C::kBlk + lane;
          int phys = -1;  // a block past the sequence: an out-of-range box, filled with zeros
          if (lb < nblk_valid) {
            phys = __ldg(row + lb);
            if (phys < 0 || phys >= a.num_blocks) {
              raise_flag(a.status, PA_FLAG_BLOCK_RANGE);
              phys = -1;
            }
          }
          uint8_t* ks = smem + C::kStageOff + st * C::kStageB;
          uint8_t* vs = ks + C::kKB;
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {
            tma_load_4d(ks + h * kBN * 128 + lane * BS * 128, &kmap, &kv_full[st], h * 64, hk, 0, phys);
            tma_load_4d(vs + h * kBN * 128 + lane * BS * 128, &vmap, &kv_full[st], h * 64, hk, 0, phys);
          }
        }
      }
    }
    // Before the CTA exits no copy may still be landing in its shared memory:
    // the last load of every stage and the last Q load (default bound).
    if (lane == 0) {
      for (uint32_t i = kt > static_cast<uint32_t>(NST) ? kt - NST : 0; i < kt; ++i)
        mbar_drain(&kv_full[i % NST], (i / NST) & 1, a.status);
      if (nq > 0) mbar_drain(q_full, (nq - 1) & 1, a.status);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ================= MMA issue (lane 0; the whole warp zeroes stale V rows)
    // Per key tile: S of both Q tiles (once their softmax warps hold the
    // previous S in registers), then the P.V products of the previous tile
    // once the softmax warps have written its P. The tensor pipe thus always
    // holds the next scores while the softmax of the current ones runs.
    bool ok = true;
    uint32_t kt = 0, nq = 0;
    uint32_t cnt[2] = {0, 0};  // S / P.V products issued per Q tile
    auto wait1 = [&](uint64_t* bar, uint32_t parity) {
      bool r = true;
      if (lane == 0) r = mbar_wait(bar, parity, a.status, a.wait_limit_ns);
      return __shfl_sync(0xffffffffu, r, 0) != 0;
    };
    // O_i += P_i V for the tile in stage st whose products are numbered c[i]
    auto issue_pv = [&](uint32_t st, const bool* act, const uint32_t* c, bool* first) {
#pragma unroll
      for (int qi = 0; qi < 2; ++qi) {
        if (!act[qi]) continue;
        const uint32_t bb = c[qi] & 1;
        if (!wait1(&p_full[qi * 2 + bb], (c[qi] >> 1) & 1)) return false;
        if (lane == 0) {
          tc::fence_after_sync();
          const uint32_t v_addr = smem_u32(smem + C::kStageOff + st * C::kStageB + C::kKB);
          const uint32_t p_t = tmem + C::kPCol + qi * 64 + bb * 32;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            tc::mma_bf16_ta(tmem + C::kOCol + qi * D, p_t + kk * 8,
                            tc::sw128_desc(v_addr + kk * 16 * 128, kBN * 128, 1024), C::kIdescO,
                            !first[qi] || kk > 0);
          tc::commit(&pv_done[qi * 2 + bb]);
        }
        first[qi] = false;
      }
      if (lane == 0) tc::commit(&kv_empty[st]);
      return true;
    };
    for (int64_t b = beg; b < end && ok;) {
      PSeg g;
      locate<GH>(b, beg, end, cta, prefix, S, HGp, a, g);
      b += g.j_hi - g.j_lo;
      if (!(ok = wait1(q_full, nq & 1))) break;
      ++nq;
      const uint32_t q_addr = smem_u32(smem);
      bool first[2] = {true, true};
      bool pact[2] = {false, false};
      uint32_t pc[2] = {0, 0}, pst = 0;
      bool have_prev = false;
      for (int j = g.j_lo; j < g.j_hi; ++j, ++kt) {
        const uint32_t st = kt % NST;
        if (!(ok = wait1(&kv_full[st], (kt / NST) & 1))) break;
        const bool act[2] = {j < g.nt0, g.t1};
        const uint32_t k_addr = smem_u32(smem + C::kStageOff + st * C::kStageB);
#pragma unroll
        for (int qi = 0; qi < 2; ++qi) {
          if (!act[qi] || !ok) continue;
          const uint32_t c = cnt[qi];
          // the softmax warps hold the previous S of this Q tile in registers
          if (c >= 1 && !(ok = wait1(&s_free[qi], (c - 1) & 1))) break;
          if (lane == 0) {
            tc::fence_after_sync();
            const uint32_t qa0 = q_addr + qi * C::kQTileB;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off_q = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
              const uint32_t off_k = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
              tc::mma_bf16(tmem + qi * 64, tc::sw128_desc(qa0 + off_q, 16, 1024),
                           tc::sw128_desc(k_addr + off_k, 16, 1024), C::kIdescS, kk > 0);
            }
            tc::commit(&s_full[qi]);
          }
        }
        if (!ok) break;
        if (j == g.j_hi - 1 && lane == 0) tc::commit(q_empty);  // Q is free once these scores are done
        // keys at or beyond L inside this tile: zero their stale V rows
        const int kbase = j * kBN;
        if (g.L - kbase < kBN) {
          const int z0 = g.L - kbase;
          const int z1 = min(kBN, (g.L + BS - 1) / BS * BS - kbase);
          uint8_t* vs = smem + C::kStageOff + st * C::kStageB + C::kKB;
          const int n16 = (z1 - z0) * 8;  // 16-byte chunks per half
          for (int i = lane; i < n16 * C::kHalves; i += 32) {
            const int h = i / n16, rem = i - h * n16;
            *reinterpret_cast<uint4*>(vs + h * kBN * 128 + (z0 + rem / 8) * 128 + (rem & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (have_prev && !(ok = issue_pv(pst, pact, pc, first))) break;
        have_prev = true;
        pst = st;
#pragma unroll
        for (int qi = 0; qi < 2; ++qi) {
          pact[qi] = act[qi];
          pc[qi] = cnt[qi];
          cnt[qi] += act[qi] ? 1 : 0;
        }
      }
      if (ok && have_prev) ok = issue_pv(pst, pact, pc, first);
    }
    // no MMA may be in flight when TMEM is released
    if (lane == 0) {
      tc::commit(mma_done);
      mbar_drain(mma_done, 0, a.status);
    }
    __syncwarp();
  } else {
    // ================= softmax: warps 4 qi .. 4 qi + 3 own Q tile qi, one row per thread
    const int qi = warp >> 2;
    const int r = tid & 127;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t o_col = C::kOCol + qi * D;
    uint32_t cnt = 0;
    bool failed = false;
    for (int64_t b = beg; b < end && !failed;) {
      PSeg g;
      locate<GH>(b, beg, end, cta, prefix, S, HGp, a, g);
      b += g.j_hi - g.j_lo;
      const int tok = g.pt * C::kPairTok + qi * C::kTOK + r / GH;
      const int lim = min(g.L - g.ql + tok, g.L - 1);  // last key this row may see
      const int jend = qi == 0 ? min(g.j_hi, g.nt0) : (g.t1 ? g.j_hi : g.j_lo);
      float m_used = -CUDART_INF_F, l = 0.f;
      int done = 0;
      for (int j = g.j_lo; j < jend; ++j) {
        const uint32_t bb = cnt & 1;
        failed = !mbar_wait(&s_full[qi], cnt & 1, a.status, a.wait_limit_ns);
        if (__any_sync(0xffffffffu, failed)) {
          failed = true;
          break;
        }
        tc::fence_after_sync();
        float sv[kBN];
        tc::ld32(t_lane + qi * 64, sv);
        tc::ld32(t_lane + qi * 64 + 32, sv + 32);
        tc::wait_ld();
        // S is in registers: the next scores of this Q tile may be computed now
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[qi]);
        const int kbase = j * kBN;
        // With a positive scale the row max is taken on the raw scores and the
        // scale is folded into the exponent's FMA below; the causal mask is
        // applied only on tiles that reach past this row's last visible key.
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
        const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * sc;
        // Rescale only when the running max grows by more than 2^8; otherwise
        // keep the old reference so P stays below 2^8 and O needs no update.
        const float m_new = fmaxf(m_used, mx);
        float alpha = 1.f;
        const bool bump = m_new > m_used + kRescaleLog2;
        if (bump) {
          alpha = fast_exp2(m_used - m_new);
          m_used = m_new;
        }
        if (done > 0 && __any_sync(0xffffffffu, bump)) {
          // O holds the P.V products up to the previous tile: wait, then rescale
          const uint32_t pb = (cnt - 1) & 1;
          failed = !mbar_wait(&pv_done[qi * 2 + pb], ((cnt - 1) >> 1) & 1, a.status, a.wait_limit_ns);
          if (__any_sync(0xffffffffu, failed)) {
            failed = true;
            break;
          }
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
        // a row that sees no key of this segment yet keeps m = -inf: its
        // probabilities are exactly 0 (exp2 of -inf)
        const float m_e = m_used == -CUDART_INF_F ? 0.f : m_used;
        uint32_t pk[kBN / 2];
        float lq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < kBN / 2; ++i) {
          const float p0 = fast_exp2(fmaf(sv[2 * i], sc, -m_e));
          const float p1 = fast_exp2(fmaf(sv[2 * i + 1], sc, -m_e));
          lq[i & 3] += p0 + p1;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        l += (lq[0] + lq[1]) + (lq[2] + lq[3]);
        if (cnt >= 2) {  // P buffer bb was last read by P.V product cnt - 2
          failed = !mbar_wait(&pv_done[qi * 2 + bb], ((cnt - 2) >> 1) & 1, a.status, a.wait_limit_ns);
          if (__any_sync(0xffffffffu, failed)) {
            failed = true;
            break;
          }
        }
        tc::st32u(t_lane + C::kPCol + qi * 64 + bb * 32, pk);
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[qi * 2 + bb]);
        ++cnt;
        ++done;
      }
      if (failed) break;
      if (done > 0) {
        const uint32_t pb = (cnt - 1) & 1;
        failed = !mbar_wait(&pv_done[qi * 2 + pb], ((cnt - 1) >> 1) & 1, a.status, a.wait_limit_ns);
        if (__any_sync(0xffffffffu, failed)) {
          failed = true;
          break;
        }
        tc::fence_after_sync();
      }
      // ---- epilogue: O / l to the output rows, or this CTA's partial
      const bool row_ok = tok < g.ql;
      const int hq = g.hg * GH + r % GH;
      if (g.slot < 0) {
        const float inv_l = 1.f / l;
        __nv_bfloat16* orow =
            static_cast<__nv_bfloat16*>(a.out) + (static_cast<size_t>(g.r0 + tok) * a.num_q_heads + hq) * D;
#pragma unroll 1
        for (int q = 0; q < D / 32; ++q) {
          float ov[32];
          tc::ld32(t_lane + o_col + 32 * q, ov);
          tc::wait_ld();
          if (row_ok) {
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
      } else {
        const size_t srow = static_cast<size_t>(g.slot) * 256 + qi * 128 + r;
        const bool has = done > 0 && l > 0.f;
        if (row_ok) a.pf_lse[srow] = has ? m_used + log2f(l) : -CUDART_INF_F;
        if (done > 0) {
          const float inv_l = has ? 1.f / l : 0.f;
#pragma unroll 1
          for (int q = 0; q < D / 32; ++q) {
            float ov[32];
            tc::ld32(t_lane + o_col + 32 * q, ov);
            tc::wait_ld();
            if (row_ok && has) {
              float* po = a.pf_o + srow * D + 32 * q;
#pragma unroll
              for (int v4 = 0; v4 < 8; ++v4)
                *reinterpret_cast<float4*>(po + 4 * v4) = make_float4(
                    ov[4 * v4] * inv_l, ov[4 * v4 + 1] * inv_l, ov[4 * v4 + 2] * inv_l, ov[4 * v4 + 3] * inv_l);
            }
          }
        }
      }
      // O is overwritten by the next segment's first P.V product, which the
      // MMA warp issues only after this Q tile's warps hand over that tile's P.
      tc::fence_before_sync();
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, C::kTmemCols);
  if (tid == 0) grid_dependency_wait();  // finish no earlier than the previous grid
}

// Merge the partials of pairs split between CTAs: block x handles the pair
// that CTA x starts and CTA x + 1 continues (if any); blockIdx.y selects 32 of
// its 256 rows; 8 threads share a row. O = sum_k 2^(lse_k - M) O_k / sum_k 2^(lse_k - M).
template <int D, int GH>
__global__ void __launch_bounds__(256) prefill_combine_kernel(const PrefillArgs a) {
  constexpr int TOK = 128 / GH, PT = 2 * TOK, kCols = D / 8;
  grid_dependency_wait();  // the prefill grid (partials and the partition) is complete
  const int S = a.num_seqs;
  const int* prefix = a.pf_prefix;
  const int Geff = prefix[S + 1], T = prefix[S + 2];
  const int c = blockIdx.x;
  if (c + 1 >= Geff) return;
  const int64_t beg = static_cast<int64_t>(c) * T / Geff, end = static_cast<int64_t>(c + 1) * T / Geff;
  PSeg g;
  locate<GH>(end - 1, beg, end, c, prefix, S, a.num_q_heads / GH, a, g);
  const int64_t ps = (end - 1) - g.j_lo;  // the pair's first and one-past-last global tile
  const int64_t pe = ps + g.nt;
  if (pe <= end || ps < beg) return;      // not split after this CTA, or not started by it
  const int c1 = cta_of_block(pe - 1, T, Geff);
  const int row = blockIdx.y * 32 + (threadIdx.x >> 3);
  const int qi = row >> 7, rr = row & 127;
  const int tok = g.pt * PT + qi * TOK + rr / GH;
  if (tok >= g.ql) return;
  const int col0 = (threadIdx.x & 7) * kCols;
  float M = -CUDART_INF_F, sum = 0.f, acc[kCols];
#pragma unroll
  for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
  for (int cc = c; cc <= c1; ++cc) {
    const int slot = cc == c ? 2 * c + (ps > beg ? 1 : 0) : 2 * cc;
    const size_t sr = static_cast<size_t>(slot) * 256 + row;
    const float lse = a.pf_lse[sr];
    if (lse == -CUDART_INF_F) continue;
    float v[kCols];
#pragma unroll
    for (int i = 0; i < kCols / 4; ++i) {
      const float4 f = *reinterpret_cast<const float4*>(a.pf_o + sr * D + col0 + 4 * i);
      v[4 * i] = f.x;
      v[4 * i + 1] = f.y;
      v[4 * i + 2] = f.z;
      v[4 * i + 3] = f.w;
    }
    const float m_new = fmaxf(M, lse);
    const float keep = fast_exp2(M - m_new), w = fast_exp2(lse - m_new);
    sum = fmaf(sum, keep, w);
#pragma unroll
    for (int i = 0; i < kCols; ++i) acc[i] = fmaf(acc[i], keep, w * v[i]);
    M = m_new;
  }
  const float inv = 1.f / sum;
  __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) +
                        (static_cast<size_t>(g.r0 + tok) * a.num_q_heads + g.hg * GH + rr % GH) * D + col0;
#pragma unroll
  for (int i = 0; i < kCols / 8; ++i) {
    uint32_t pk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[8 * i + 2 * k] * inv, acc[8 * i + 2 * k + 1] * inv);
      pk[k] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(orow + 8 * i) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

template <int D, int BS, int GH>
cudaError_t launch_prefill_t(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, cudaStream_t stream) {
  using C = PrefillCfg<D, BS, GH>;
  auto kern = paged_prefill_kernel<D, BS, GH>;
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
  log_launch("paged_prefill_kernel", a.grid, kThreads, smem, 1);
  e = launch_chained(kern, dim3(a.grid), dim3(kThreads), smem, stream, qmap, kmap, vmap, a);
  if (e != cudaSuccess) return e;
  return launch_chained(prefill_combine_kernel<D, GH>, dim3(a.grid, 8), dim3(256), 0, stream, a);
}

template <int D, int BS>
cudaError_t launch_prefill_gh(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, int gh, cudaStream_t stream) {
  switch (gh) {
    case 16: return launch_prefill_t<D, BS, 16>(a, qmap, kmap, vmap, stream);
    case 8: return launch_prefill_t<D, BS, 8>(a, qmap, kmap, vmap, stream);
    case 4: return launch_prefill_t<D, BS, 4>(a, qmap, kmap, vmap, stream);
    case 2: return launch_prefill_t<D, BS, 2>(a, qmap, kmap, vmap, stream);
    default: return launch_prefill_t<D, BS, 1>(a, qmap, kmap, vmap, stream);
  }
}

template <int D>
cudaError_t launch_prefill_bs(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, int bs, int gh, cudaStream_t stream) {
  switch (bs) {
    case 8: return launch_prefill_gh<D, 8>(a, qmap, kmap, vmap, gh, stream);
    case 16: return launch_prefill_gh<D, 16>(a, qmap, kmap, vmap, gh, stream);
    default: return launch_prefill_gh<D, 32>(a, qmap, kmap, vmap, gh, stream);
  }
}

}  // namespace

int32_t prefill_heads_per_tile(int32_t group) {
  return (group <= 16 && (group & (group - 1)) == 0) ? group : 1;
}

int32_t prefill_grid(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_query_len,
                     int32_t max_context_len) {
  const int64_t gh = prefill_heads_per_tile(num_q_heads / num_kv_heads);
  const int64_t pair_tok = 2 * (128 / gh);
  const int64_t pairs = static_cast<int64_t>(num_seqs) * (num_q_heads / gh) * ((max_query_len + pair_tok - 1) / pair_tok);
  const int64_t tiles = pairs * ((static_cast<int64_t>(max_context_len) + kBN - 1) / kBN);
  int64_t g = (tiles + kMinTilesPerCta - 1) / kMinTilesPerCta;
  if (g > num_sms()) g = num_sms();
  return static_cast<int32_t>(g < 1 ? 1 : g);
}

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                           const CUtensorMap& vmap, const pa_cache_desc& c, cudaStream_t stream) {
  if (c.dtype != PA_BF16) return cudaErrorNotSupported;
  const int gh = prefill_heads_per_tile(a.num_q_heads / a.num_kv_heads);
  if (c.head_dim == 64) return launch_prefill_bs<64>(a, qmap, kmap, vmap, c.block_size, gh, stream);
  return launch_prefill_bs<128>(a, qmap, kmap, vmap, c.block_size, gh, stream);
}

}  // namespace pa
