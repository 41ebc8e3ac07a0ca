// Paged decode attention (query rows with q_len == 1), split over the block
// table with an online softmax, plus the kernel that merges split rows.
//
// What is computed: for sequence s with L = context_lens[s] keys and query
// head h, o = softmax(q . K[0:L]^T * scale) . V[0:L], where key i lives in
// row i % bs of physical block block_tables[s][i / bs] for KV head
// h / (Hq / Hkv). The logical-to-physical walk is the page table of
// "vLLM核心架构：PagedAttention原理、KV Cache管理、连续批处理机制",
// §"一、PagedAttention：虚拟内存的灵感"; the decode call is the one the page
// "深入解析 nano-vLLM 推理引擎的分页 KV 缓存与内存优化架构",
// §"工程落地：配置参数与监控指标" hands to a library. Decode is bound by memory
// bandwidth (§"三、连续批处理：让GPU一刻不停" of the first page), which shapes
// the design.
//
// This CUDA-core kernel serves every decode call by default: both dtypes,
// head_dim 64 and 128, grouped and ungrouped heads, and the suffix pass of
// cascade decode. A tensor-core variant for grouped bf16 heads of 128
// (decode_tc.cu, same partition and merge) is selected only on request
// (environment PA_DECODE_TC=1).
//
// Design (B200):
//  * A unit is (sequence, group of GH query heads sharing one KV head); its
//    work is the sequence's ceil(L/bs) KV blocks of that head. All units'
//    blocks are numbered contiguously (unit-major) and the persistent grid of
//    G CTAs splits that range evenly: CTA c takes blocks [c*B/G, (c+1)*B/G).
//    Every CTA streams the same number of blocks, so there is no tail, and a
//    CTA touches only a few units (segments).
//  * One producer warp gathers each KV block of the current head with two TMA
//    tensor loads (K, V: box {D, 1, bs, 1}) into a ring of NST shared-memory
//    stages; the ring runs on across segments.
//  * NCW consumer warps take the ring's blocks round-robin. LPR lanes hold one
//    16-byte slice each of a key row (TPW rows per warp step). q.k uses packed
//    fp32x2 FMAs; the per-head partial sums are reduce-scattered across the
//    row's lanes so each lane ends with one head's full score, does that
//    head's exp, and the lanes exchange probabilities for P.V. Warps merge
//    their (m, l, acc) through shared memory at the end of a segment.
//  * GQA: every KV block is read once for the GH query heads of its group.
//    Without grouping and with Hkv a multiple of 4, a unit is 4 adjacent KV
//    heads: one box {D, 4, bs, 1} reads 4*D contiguous elements per token and
//    consumer warp w owns head w of every block.
//  * Cascade decode: a sequence's first skip_blocks[s] blocks are left to the
//    prefix pass; its units stream the rest and always leave a partial.
//  * Keys at or beyond L (the unfilled tail of the last block) are masked and
//    their V rows are never read, so stale bits there (even NaN) cannot leak.
//  * A unit covered by one CTA writes its output rows directly. Otherwise each
//    covering CTA c writes (o / l, m + log2 l) to partial slot u + c (unique:
//    the CTAs covering unit u+1 start where those of unit u end), and a second
//    kernel merges them: O = sum_c 2^(lse_c - M) O_c / sum_c 2^(lse_c - M).
#include <math_constants.h>

#include "decode_common.cuh"
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

// KH > 1 (only with GH == 1, KH == NCW): the CTA streams KH adjacent KV heads
// at once -- one TMA box {D, KH, bs, 1} reads KH*D contiguous elements per
// token -- and consumer warp w owns head w of every block.
template <typename T, int D, int BS, int GH, int KH, int NCW>
struct DecodeCfg {
  static constexpr int kEB = sizeof(T);
  static constexpr int kRowB = D * kEB;             // bytes of one key row (one head)
  static constexpr int kLPR = kRowB / 16;           // lanes per row
  static constexpr int kTPW = 32 / kLPR;            // rows per warp step
  static constexpr int kEPL = 16 / kEB;             // elements per lane
  static constexpr int kSteps = BS / kTPW;          // warp steps per block
  static constexpr int kNIT = kSteps < 16 ? kSteps : 16;  // steps per softmax update
  static constexpr int kNUPD = kSteps / kNIT;
  static constexpr int kLogLPR = kLPR == 32 ? 5 : (kLPR == 16 ? 4 : 3);
  static constexpr int kLogGH = GH == 4 ? 2 : (GH == 2 ? 1 : 0);
  static constexpr int kHeadShift = kLogLPR - kLogGH;  // lane bits below the head index
  static constexpr int kPairs = kEPL / 2;              // fp32 pairs per lane
  static constexpr int kHPU = GH * KH;                 // query heads per unit
  static constexpr int kTokB = KH * kRowB;             // bytes per token in a stage
  static constexpr int kStageB = 2 * BS * kTokB;       // K block + V block
  // Stages: about 64 KiB in flight per CTA (3 CTAs per SM keep ~192 KiB of
  // HBM reads outstanding), and a multiple of NCW so that every use of a stage
  // belongs to the same consumer warp (its parity waits then never run more
  // than one phase ahead).
  // With KH > 1 every warp reads every stage, so any count works; ~96 KiB.
  static constexpr int kNST0 = 65536 / kStageB;
  static constexpr int kNST1 = kNST0 < NCW ? NCW : (kNST0 > 16 ? 16 : kNST0);
  static constexpr int kNSTM = 98304 / kStageB;
  static constexpr int kNST = KH > 1 ? (kNSTM < 2 ? 2 : (kNSTM > 8 ? 8 : kNSTM)) : (kNST1 / NCW) * NCW;
  static constexpr int kThreads = (NCW + 1) * 32;
  static constexpr int kCombFloats = KH > 1 ? 0 : NCW * GH * (D + 2);
  // dynamic smem: stages | bars | comb | warp totals | abort | seq prefix, clen, row
  static constexpr int kBarOff = kNST * kStageB;
  static constexpr int kCombOff = kBarOff + 2 * kNST * 8;
  static constexpr int kScanOff = kCombOff + kCombFloats * 4;
  static constexpr int kAbortOff = kScanOff + 32 * 4;
  static constexpr int kSeqOff = kAbortOff + 16;
  static_assert(kRowB % 16 == 0 && 32 % kLPR == 0, "row must split into lanes");
  static_assert(BS % kTPW == 0 && kSteps % kNIT == 0, "block must split into steps");
  static_assert(KH > 1 || kNST % NCW == 0, "each stage must always go to the same consumer warp");
  static_assert(KH == 1 || (GH == 1 && KH == NCW), "multi-head CTAs: one warp per KV head");
  static_assert(kLogGH <= kLogLPR, "more heads than lanes per row");
  static size_t smem_bytes(int num_seqs) { return 1024 + kSeqOff + 12ull * (num_seqs + 1); }
};

#ifndef PA_DECODE_GQA_CTAS_PER_SM
#define PA_DECODE_GQA_CTAS_PER_SM 3
#endif

template <typename T, int D, int BS, int GH, int KH, int NCW>
// Registers are budgeted for 4 (one head) or PA_DECODE_GQA_CTAS_PER_SM
// (grouped heads) CTAs per SM: more resident warps hide the latency of the
// shuffle and FMA chains.
__global__ void __launch_bounds__((NCW + 1) * 32, (GH == 1 ? 4 : PA_DECODE_GQA_CTAS_PER_SM))
    paged_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const DecodeArgs a) {
  using C = DecodeCfg<T, D, BS, GH, KH, NCW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + C::kNST;
  float* comb = reinterpret_cast<float*>(smem + C::kCombOff);
  int* warp_tot = reinterpret_cast<int*>(smem + C::kScanOff);
  volatile int* abort_word = reinterpret_cast<volatile int*>(smem + C::kAbortOff);
  int* prefix = reinterpret_cast<int*>(smem + C::kSeqOff);      // [S+1] decode blocks before seq s
  int* clen = prefix + (a.num_seqs + 1);                         // [S]
  int* qrow = clen + a.num_seqs;                                 // [S]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.num_q_heads / a.num_kv_heads;
  const int HG = a.num_q_heads / C::kHPU;  // units per sequence

  if (tid == 0) {
    for (int i = 0; i < C::kNST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], KH > 1 ? NCW : 1);  // KH > 1: every consumer warp releases
    }
    fence_barrier_init();
    *abort_word = 0;
  }
  if (warp == NCW && lane == 0) {
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
      clen[s] = L;
      qrow[s] = r0;
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
  __syncthreads();
  // The grids chained after this one may start now: every input they read
  // was complete before this grid passed its wait, and each of them waits
  // for its own predecessor at most.
  launch_dependents();
  const int64_t B = static_cast<int64_t>(prefix[a.num_seqs]) * HG;  // blocks of all units
  if (blockIdx.x == 0 && a.seq_prefix)
    for (int i = tid; i <= a.num_seqs; i += blockDim.x) a.seq_prefix[i] = prefix[i];
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * B / a.grid;
  const int64_t end = static_cast<int64_t>(blockIdx.x + 1) * B / a.grid;

  // the segment of this CTA that starts at global block b (beg <= b < end)
  auto segment_at = [&](int64_t b, Segment& g) {
    locate_segment(b, prefix, a.num_seqs, HG, beg, end, static_cast<int>(blockIdx.x), g);
    apply_skip(a.skip_blocks, HG, static_cast<int>(blockIdx.x), g);
    g.L = clen[g.s];
  };

  if (warp == NCW) {
    // ================= producer warp: TMA gathers of K/V blocks
    // The block ids of the next segment are fetched while the current
    // segment's loads are issued, so a segment never waits on a table read.
    auto fetch_ids = [&](const Segment& g, int b0) {  // raw ids; checked when used
      return b0 + lane < g.bhi
                 ? __ldg(a.block_tables + static_cast<size_t>(g.s) * a.max_blocks_per_seq + g.skip + b0 + lane)
                 : 0;
    };
    auto checked = [&](int phys) {
      if (phys < 0 || phys >= a.num_blocks) {
        raise_flag(a.status, PA_FLAG_BLOCK_RANGE);
        return -1;  // a fully out-of-bounds box: TMA fills zeros, reads nothing
      }
      return phys;
    };
    uint32_t k = 0;
    bool ok = true;
    Segment cur, nxt;
    int64_t b = beg;
    int ids = 0;
    if (b < end) {
      segment_at(b, cur);
      ids = fetch_ids(cur, cur.blo);
    }
    while (b < end && ok) {
      const int64_t bn = b + (cur.bhi - cur.blo);
      int nids = 0;
      if (bn < end) {
        segment_at(bn, nxt);
        nids = fetch_ids(nxt, nxt.blo);
      }
      const int hk = (cur.hg * C::kHPU) / G;  // first KV head of the unit
      for (int b0 = cur.blo; b0 < cur.bhi && ok; b0 += 32) {
        int cur_ids = checked(b0 == cur.blo ? ids : fetch_ids(cur, b0));
        const int cnt = min(32, cur.bhi - b0);
        for (int i = 0; i < cnt; ++i, ++k) {
          const int pb = __shfl_sync(0xffffffffu, cur_ids, i);
          int good = 1;
          if (lane == 0) {
            const uint32_t st = k % C::kNST, use = k / C::kNST;
            good = mbar_wait(&empty[st], (use & 1) ^ 1, a.status, a.wait_limit_ns);
            if (good) {
              uint8_t* dst = smem + st * C::kStageB;
              mbar_arrive_expect_tx(&full[st], C::kStageB);
              tma_load_4d(dst, &kmap, &full[st], 0, hk, 0, pb);
              tma_load_4d(dst + BS * C::kTokB, &vmap, &full[st], 0, hk, 0, pb);
            }
          }
          ok = __shfl_sync(0xffffffffu, good, 0) != 0;
          if (!ok) break;
        }
      }
      cur = nxt;
      ids = nids;
      b = bn;
    }
    // Every load this warp issued lands before it exits (the last one of each
    // stage; default bound), so no copy is still writing into shared memory
    // when the CTA exits, even if the consumers gave up early.
    if (lane == 0)
      for (uint32_t i = k > static_cast<uint32_t>(C::kNST) ? k - C::kNST : 0; i < k; ++i)
        mbar_drain(&full[i % C::kNST], (i / C::kNST) & 1, a.status);
    return;
  }

  // ================= consumer warps
  const int sub = lane / C::kLPR;  // which row of a warp step
  const int c = lane % C::kLPR;    // which 16-byte slice of the row
  uint32_t k = 0;
  for (int64_t b = beg; b < end;) {
    Segment g;
    segment_at(b, g);
    b += g.bhi - g.blo;
    const int blo = g.blo;
    const int nblk = g.bhi - g.blo;
    const int h0 = g.hg * C::kHPU + (KH > 1 ? warp : 0);  // first query head of this warp
    const int row = qrow[g.s];
    const int L = g.L;
    // q (pre-multiplied by scale * log2 e) as fp32 pairs for every head of the group
    float2 q2[GH][C::kPairs];
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
#pragma unroll
    for (int g = 0; g < GH; ++g) {
      const uint4 qv = *reinterpret_cast<const uint4*>(
          static_cast<const uint8_t*>(a.q) +
          ((static_cast<size_t>(row) * a.num_q_heads + h0 + g) * D + c * C::kEPL) * C::kEB);
      Elem<T>::widen2(qv, q2[g]);
#pragma unroll
      for (int i = 0; i < C::kPairs; ++i) q2[g][i] = __fmul2_rn(q2[g][i], sc2);
    }
    // After the reduce-scatter below this lane holds the full score of one
    // head of the group (hsel); m and l track that head.
    const int hsel = (c >> C::kHeadShift) & (GH - 1);
    float m = -CUDART_INF_F, l = 0.f;
    float2 acc2[GH][C::kPairs];
#pragma unroll
    for (int g = 0; g < GH; ++g)
#pragma unroll
      for (int i = 0; i < C::kPairs; ++i) acc2[g][i] = make_float2(0.f, 0.f);

    bool ok = true;
    const int first = KH > 1 ? 0 : (warp - static_cast<int>(k % NCW) + NCW) % NCW;
    for (int i = first; i < nblk; i += (KH > 1 ? 1 : NCW)) {
      const uint32_t kk = k + i;
      const uint32_t st = kk % C::kNST;
      if (!mbar_wait(&full[st], (kk / C::kNST) & 1, a.status, a.wait_limit_ns)) { ok = false; break; }
      const uint8_t* Ks = smem + st * C::kStageB + (KH > 1 ? warp * C::kRowB : 0);
      const uint8_t* Vs = Ks + BS * C::kTokB;
      const int tok0 = (g.skip + blo + i) * BS;
#pragma unroll
      for (int u = 0; u < C::kNUPD; ++u) {
        float sc[C::kNIT];
#pragma unroll
        for (int it = 0; it < C::kNIT; ++it) {
          const int t = (u * C::kNIT + it) * C::kTPW + sub;
          const uint4 kv = *reinterpret_cast<const uint4*>(Ks + t * C::kTokB + c * 16);
          float2 k2[C::kPairs];
          Elem<T>::widen2(kv, k2);
          float v[GH];
#pragma unroll
          for (int g = 0; g < GH; ++g) {
            float2 d2 = __fmul2_rn(q2[g][0], k2[0]);
#pragma unroll
            for (int e = 1; e < C::kPairs; ++e) d2 = __ffma2_rn(q2[g][e], k2[e], d2);
            v[g] = d2.x + d2.y;
          }
          // reduce-scatter over the head bits of c: each level halves the
          // heads a lane keeps and adds the partner's half
#pragma unroll
          for (int lvl = 0; lvl < C::kLogGH; ++lvl) {
            const int off = C::kLPR >> (lvl + 1);
            const bool up = (c & off) != 0;
            const int half = GH >> (lvl + 1);
#pragma unroll
            for (int h = 0; h < half; ++h) {
              const float keep = up ? v[half + h] : v[h];
              const float send = up ? v[h] : v[half + h];
              v[h] = keep + __shfl_xor_sync(0xffffffffu, send, off);
            }
          }
          float s1 = v[0];
#pragma unroll
          for (int off = C::kLPR >> (C::kLogGH + 1); off > 0; off >>= 1) s1 += __shfl_xor_sync(0xffffffffu, s1, off);
          sc[it] = tok0 + t < L ? s1 : -CUDART_INF_F;
        }
        float mx = sc[0];
#pragma unroll
        for (int it = 1; it < C::kNIT; ++it) mx = fmaxf(mx, sc[it]);
#pragma unroll
        for (int off = C::kLPR; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m, mx);
        const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
        const float alpha = fast_exp2(m - m_use);
        m = m_new;
        l *= alpha;
#pragma unroll
        for (int it = 0; it < C::kNIT; ++it) {
          const float p = fast_exp2(sc[it] - m_use);
          sc[it] = p;
          l += p;
        }
#pragma unroll
        for (int g = 0; g < GH; ++g) {
          const float ag = GH == 1 ? alpha : __shfl_sync(0xffffffffu, alpha, g << C::kHeadShift);
          const float2 ag2 = make_float2(ag, ag);
#pragma unroll
          for (int e = 0; e < C::kPairs; ++e) acc2[g][e] = __fmul2_rn(acc2[g][e], ag2);
        }
#pragma unroll
        for (int it = 0; it < C::kNIT; ++it) {
          const int t = (u * C::kNIT + it) * C::kTPW + sub;
          // rows at or beyond L are never read (stale bits may be NaN); their p is 0
          const uint4 vv = tok0 + t < L ? *reinterpret_cast<const uint4*>(Vs + t * C::kTokB + c * 16)
                                        : make_uint4(0u, 0u, 0u, 0u);
          float2 v2[C::kPairs];
          Elem<T>::widen2(vv, v2);
#pragma unroll
          for (int g = 0; g < GH; ++g) {
            const float pg = GH == 1 ? sc[it] : __shfl_sync(0xffffffffu, sc[it], sub * C::kLPR + (g << C::kHeadShift));
            const float2 p2 = make_float2(pg, pg);
#pragma unroll
            for (int e = 0; e < C::kPairs; ++e) acc2[g][e] = __ffma2_rn(v2[e], p2, acc2[g][e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    k += nblk;
    if (!ok) *abort_word = 1;  // still take part in the barrier below

    // ---- merge the rows of this warp (lanes with the same slice c)
#pragma unroll
    for (int off = C::kLPR; off < 32; off <<= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
      for (int g = 0; g < GH; ++g)
#pragma unroll
        for (int e = 0; e < C::kPairs; ++e) {
          acc2[g][e].x += __shfl_xor_sync(0xffffffffu, acc2[g][e].x, off);
          acc2[g][e].y += __shfl_xor_sync(0xffffffffu, acc2[g][e].y, off);
        }
    }
    if constexpr (KH > 1) {
      // this warp's head is complete (no other warp saw it): write it
      if (!ok) return;
      if (sub == 0) {
        const float inv_l = 1.f / l;
        if (g.slot < 0) {
          T* o = static_cast<T*>(a.out) + (static_cast<size_t>(row) * a.num_q_heads + h0) * D + c * C::kEPL;
#pragma unroll
          for (int e = 0; e < C::kPairs; ++e) {
            o[2 * e] = Elem<T>::narrow(acc2[0][e].x * inv_l);
            o[2 * e + 1] = Elem<T>::narrow(acc2[0][e].y * inv_l);
          }
        } else {
          const size_t part = static_cast<size_t>(g.slot) * C::kHPU + warp;
          float* po = a.part_o + part * D + c * C::kEPL;
#pragma unroll
          for (int e = 0; e < C::kPairs; ++e) {
            po[2 * e] = acc2[0][e].x * inv_l;
            po[2 * e + 1] = acc2[0][e].y * inv_l;
          }
          if (c == 0) a.part_lse[part] = m + log2f(l);
        }
      }
      continue;
    }
    float* cb = comb + warp * GH * (D + 2);
    if (sub == 0) {
#pragma unroll
      for (int g = 0; g < GH; ++g)
#pragma unroll
        for (int e = 0; e < C::kPairs; ++e) {
          cb[g * (D + 2) + c * C::kEPL + 2 * e] = acc2[g][e].x;
          cb[g * (D + 2) + c * C::kEPL + 2 * e + 1] = acc2[g][e].y;
        }
      if ((c & ((1 << C::kHeadShift) - 1)) == 0) {
        cb[hsel * (D + 2) + D] = m;
        cb[hsel * (D + 2) + D + 1] = l;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
    if (*abort_word) return;  // every consumer warp sees the same value here

    // ---- merge the warps; write the output rows or this CTA's partial
    const float* cball = comb;
    for (int idx = tid; idx < GH * D; idx += NCW * 32) {
      const int gi = idx / D, d = idx - gi * D;
      float M = -CUDART_INF_F;
#pragma unroll
      for (int ww = 0; ww < NCW; ++ww) M = fmaxf(M, cball[(ww * GH + gi) * (D + 2) + D]);
      float sl = 0.f, so = 0.f;
#pragma unroll
      for (int ww = 0; ww < NCW; ++ww) {
        const float* pw = cball + (ww * GH + gi) * (D + 2);
        const float f = fast_exp2(pw[D] - M);
        sl = fmaf(pw[D + 1], f, sl);
        so = fmaf(pw[d], f, so);
      }
      const float o = so / sl;
      if (g.slot < 0) {
        static_cast<T*>(a.out)[(static_cast<size_t>(row) * a.num_q_heads + h0 + gi) * D + d] = Elem<T>::narrow(o);
      } else {
        const size_t part = static_cast<size_t>(g.slot) * GH + gi;
        a.part_o[part * D + d] = o;
        if (d == 0) a.part_lse[part] = M + log2f(sl);
      }
    }
    // the merge buffer is reused by the next segment
    asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
  }
}

// One CTA per unit (sequence, head group), GH x D threads: merge the
// partials of a unit that several CTAs streamed and, for a cascade sequence,
// the prefix-pass partials of its shared blocks, with weights
// 2^(lse_j - M) / sum_j 2^(lse_j - M). Each thread merges its own (head,
// column) with a running max, so no shared memory and no block barrier.
template <typename T, int D, int BS, int GH>  // GH here: query heads per unit
__global__ void __launch_bounds__(GH * D) decode_combine_kernel(const DecodeArgs a) {
  launch_dependents();
  grid_dependency_wait();  // the decode grid (partials and the block prefix) is complete
  const int HG = a.num_q_heads / GH;
  const int u = blockIdx.x;
  const int s = u / HG, hg = u - s * HG;
  const int nbs = a.seq_prefix[s + 1] - a.seq_prefix[s];
  const int skip = a.skip_blocks ? __ldg(a.skip_blocks + s) : 0;
  const int n1 = skip > 0 ? (skip + a.l1_chunk_blocks - 1) / a.l1_chunk_blocks : 0;  // prefix-pass chunks
  if (nbs == 0 && n1 == 0) return;
  int c0 = 0, n2 = 0;  // covering decode CTAs c0 .. c0 + n2 - 1
  if (nbs > 0) {
    const int64_t B = static_cast<int64_t>(a.seq_prefix[a.num_seqs]) * HG;
    const int64_t ub0 = static_cast<int64_t>(a.seq_prefix[s]) * HG + static_cast<int64_t>(hg) * nbs;
    c0 = cta_of_block(ub0, B, a.grid);
    n2 = cta_of_block(ub0 + nbs - 1, B, a.grid) - c0 + 1;
    if (n2 == 1 && n1 == 0) return;  // one CTA covered the unit and wrote its rows
  }
  const int n = n2 + n1;
  const int tid = threadIdx.x;
  const int gi = tid / D, d = tid - gi * D;  // this thread's (head, column)
  const size_t slot0 = static_cast<size_t>(u) + c0;
  const size_t l1_row = (static_cast<size_t>(s) * a.num_q_heads + static_cast<size_t>(hg) * GH + gi) * a.l1_max_chunks;
  const int64_t Bt = static_cast<int64_t>(a.seq_prefix[a.num_seqs]) * HG;
  // Each thread folds its partials with a running max (weights 2^(lse - M)).
  float M = -CUDART_INF_F, sum = 0.f, acc = 0.f;
  auto fold = [&](float lse, float val) {
    if (lse == -CUDART_INF_F) return;
    const float m_new = fmaxf(M, lse);
    const float keep = fast_exp2(M - m_new), w = fast_exp2(lse - m_new);
    sum = fmaf(sum, keep, w);
    acc = fmaf(acc, keep, w * val);
    M = m_new;
  };
  if (Bt >= a.grid) {
    // every CTA in [c0, c0 + n2) streamed a block of the unit and wrote its
    // partial; loads are issued four at a time, ahead of the arithmetic
    for (int j0 = 0; j0 < n2; j0 += 4) {
      float lse[4], val[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = j0 + q;
        lse[q] = -CUDART_INF_F;
        val[q] = 0.f;
        if (j < n2) {
          const size_t part = (slot0 + j) * GH + gi;
          lse[q] = a.part_lse[part];
          val[q] = a.part_o[part * D + d];
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) fold(lse[q], val[q]);
    }
  } else if (n2 > 0) {
    // more CTAs than blocks: some CTAs in [c0, c0 + n2) streamed nothing and
    // wrote no partial (their stale slots are never read); the ones that did
    // are the owners of the unit's blocks, in order
    const int64_t ub0 = static_cast<int64_t>(a.seq_prefix[s]) * HG + static_cast<int64_t>(hg) * nbs;
    int prev = -1;
    for (int k = 0; k < nbs; ++k) {
      const int c = cta_of_block(ub0 + k, Bt, a.grid);
      if (c == prev) continue;
      prev = c;
      const size_t part = (slot0 + (c - c0)) * GH + gi;
      fold(a.part_lse[part], a.part_o[part * D + d]);
    }
  }
  for (int j = n2; j < n; ++j)  // prefix-pass partials of cascade decode
    fold(a.l1_lse[l1_row + (j - n2)], a.l1_o[(l1_row + (j - n2)) * D + d]);
  const int row = __ldg(a.query_start_loc + s);
  static_cast<T*>(a.out)[(static_cast<size_t>(row) * a.num_q_heads + hg * GH + gi) * D + d] =
      Elem<T>::narrow(acc / sum);
}

constexpr int kNCW = 4;

template <typename T, int D, int BS, int GH, int KH>
cudaError_t launch_decode_t(DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            cudaStream_t stream) {
  using C = DecodeCfg<T, D, BS, GH, KH, kNCW>;
  auto kern = paged_decode_kernel<T, D, BS, GH, KH, kNCW>;
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
  const int per_sm = ctas_per_sm(reinterpret_cast<const void*>(kern), C::kThreads, smem, 8);
  int grid = num_sms() * per_sm;
  if (grid > decode_max_grid()) grid = decode_max_grid();
  // no more CTAs than the blocks there can be to stream (a CTA without a block
  // only costs its launch, and makes the merge skip over it)
  const int64_t max_blocks = static_cast<int64_t>(a.num_seqs) * (a.num_q_heads / C::kHPU) *
                             ((static_cast<int64_t>(a.max_context_len) + BS - 1) / BS);
  if (grid > max_blocks) grid = static_cast<int>(max_blocks > 0 ? max_blocks : 1);
  if (const char* env = getenv("PA_DECODE_GRID")) {  // testing / tuning: cap the grid
    const int v = atoi(env);
    if (v >= 1 && v < grid) grid = v;
  }
  a.grid = grid;
  a.hpu = C::kHPU;
  log_launch("paged_decode_kernel", grid, C::kThreads, smem, per_sm);
  return launch_chained(kern, dim3(grid), dim3(C::kThreads), smem, stream, kmap, vmap, a);
}

template <typename T, int D, int BS>
cudaError_t launch_decode_gh(DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                             const pa_cache_desc& desc, cudaStream_t stream) {
  const int group = a.num_q_heads / a.num_kv_heads;
  if (decode_kv_heads_per_cta(group, desc) == kNCW) return launch_decode_t<T, D, BS, 1, kNCW>(a, kmap, vmap, stream);
  switch (decode_heads_per_cta(group)) {
    case 4: return launch_decode_t<T, D, BS, 4, 1>(a, kmap, vmap, stream);
    case 2: return launch_decode_t<T, D, BS, 2, 1>(a, kmap, vmap, stream);
    default: return launch_decode_t<T, D, BS, 1, 1>(a, kmap, vmap, stream);
  }
}

template <typename T, int D>
cudaError_t launch_decode_bs(DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                             const pa_cache_desc& desc, cudaStream_t stream) {
  switch (desc.block_size) {
    case 8: return launch_decode_gh<T, D, 8>(a, kmap, vmap, desc, stream);
    case 16: return launch_decode_gh<T, D, 16>(a, kmap, vmap, desc, stream);
    default: return launch_decode_gh<T, D, 32>(a, kmap, vmap, desc, stream);
  }
}

template <typename T, int D, int BS, int GH>
cudaError_t launch_combine_t(const DecodeArgs& a, cudaStream_t stream) {
  auto kern = decode_combine_kernel<T, D, BS, GH>;
  const unsigned grid = static_cast<unsigned>(a.num_seqs) * (a.num_q_heads / GH);
  return launch_chained(kern, dim3(grid), dim3(GH * D), 0, stream, a);
}

template <typename T, int D, int BS>
cudaError_t launch_combine_gh(const DecodeArgs& a, const pa_cache_desc& desc, cudaStream_t stream) {
  (void)desc;
  switch (a.hpu) {  // the unit of the decode grid that was launched
    case 8: return launch_combine_t<T, D, BS, 8>(a, stream);
    case 4: return launch_combine_t<T, D, BS, 4>(a, stream);
    case 2: return launch_combine_t<T, D, BS, 2>(a, stream);
    default: return launch_combine_t<T, D, BS, 1>(a, stream);
  }
}

template <typename T, int D>
cudaError_t launch_combine_bs(const DecodeArgs& a, const pa_cache_desc& desc, cudaStream_t stream) {
  switch (desc.block_size) {
    case 8: return launch_combine_gh<T, D, 8>(a, desc, stream);
    case 16: return launch_combine_gh<T, D, 16>(a, desc, stream);
    default: return launch_combine_gh<T, D, 32>(a, desc, stream);
  }
}

}  // namespace

int32_t decode_heads_per_cta(int32_t group) {
  if (group % 4 == 0) return 4;
  if (group % 2 == 0) return 2;
  return 1;
}

int32_t decode_kv_heads_per_cta(int32_t group, const pa_cache_desc& c) {
  // 4 adjacent KV heads per CTA when there is no grouping, the heads divide
  // evenly, and two 4-head stages (K + V) fit in 128 KiB of shared memory.
  const int64_t stage = 2ll * c.block_size * kNCW * c.head_dim * (c.dtype == PA_BF16 ? 2 : 4);
  return (group == 1 && c.num_kv_heads % kNCW == 0 && stage <= 65536) ? kNCW : 1;
}

int32_t decode_heads_per_unit(int32_t group, const pa_cache_desc& c) {
  return decode_heads_per_cta(group) * decode_kv_heads_per_cta(group, c);
}

int32_t decode_max_grid() { return num_sms() * 8; }

cudaError_t launch_decode(DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          const pa_cache_desc& c, cudaStream_t stream) {
  if (c.dtype == PA_BF16) {
    if (c.head_dim == 64) return launch_decode_bs<__nv_bfloat16, 64>(a, kmap, vmap, c, stream);
    return launch_decode_bs<__nv_bfloat16, 128>(a, kmap, vmap, c, stream);
  }
  if (c.head_dim == 64) return launch_decode_bs<float, 64>(a, kmap, vmap, c, stream);
  return launch_decode_bs<float, 128>(a, kmap, vmap, c, stream);
}

cudaError_t launch_decode_combine(const DecodeArgs& a, const pa_cache_desc& c, cudaStream_t stream) {
  if (c.dtype == PA_BF16) {
    if (c.head_dim == 64) return launch_combine_bs<__nv_bfloat16, 64>(a, c, stream);
    return launch_combine_bs<__nv_bfloat16, 128>(a, c, stream);
  }
  if (c.head_dim == 64) return launch_combine_bs<float, 64>(a, c, stream);
  return launch_combine_bs<float, 128>(a, c, stream);
}

}  // namespace pa
