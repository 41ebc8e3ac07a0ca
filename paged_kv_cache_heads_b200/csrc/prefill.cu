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
//    both multiply the same K/V tiles, and their two dependency chains keep
//    the tensor pipe busy while either one's softmax runs (ping-pong).
//  * Keys come in tiles of 128: an M=128, N=128, K=16 MMA keeps the tensor
//    pipe above 90% busy where N=64 reaches about 55% (measured).
//  * Work units: a pair's key tiles plus a fixed number of units for the cost
//    of starting and finishing it (Q tiles, epilogue, pipeline refill); all
//    units are numbered contiguously (sequence, head group, pair) and the grid
//    splits the whole range evenly (stream-K): CTA c takes units
//    [c*T/G, (c+1)*T/G). A pair one CTA covers entirely is written straight to
//    the output; otherwise each covering CTA leaves a partial
//    (O / l, m + log2 l) per row, the CTA that starts the pair records which
//    CTAs cover it, and prefill_combine_kernel merges them.
//  * Warp 9 loads both Q tiles of a segment with TMA. Warps 9-12 gather each
//    key tile's K rows and warps 13-15 its V rows through the block table with
//    16-byte cp.async copies straight into the 128-byte swizzled layout of the
//    MMA operands (a tensor-copy box per KV block and 64 columns would cost one
//    serialised issue each), into a ring of K/V stages. Rows at or beyond L
//    (the unfilled tail of the last block, blocks past the sequence) are
//    filled with zeros, so stale bits there cannot reach the output.
//  * TMEM (512 columns): S_i of Q tile i in columns [128 i, 128 i + 128);
//    its softmax writes P_i as bf16 over the first 64 of them; O_i at
//    256 + i * head_dim. Warp 8 (one thread) issues, per key tile j:
//    O_0 += P_0(j-1) V(j-1), S_0(j) = Q_0 K(j)^T, then the same for tile 1.
//    The MMAs of one thread run in issue order, so S_i(j) overwrites P_i(j-1)
//    only after the product that reads it, and a completed S_i(j) implies a
//    completed O_i update for j-1. tcgen05.commit arrives on mbarriers; every
//    wait is bounded.
//  * Warps 0-3 and 4-7 run the softmax of Q tile 0 and 1: one row per thread
//    (TMEM lane = row), fp32 online softmax with exp2 on the scale folded into
//    log2 e. O is rescaled in TMEM only when a row's running max grows by
//    more than 2^8.
#include <cuda_fp16.h>
#include <math_constants.h>

#include "decode_common.cuh"
#include "pa_common.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int kBN = 128;            // keys per tile
constexpr float kRescaleLog2 = 8.f;
constexpr int kMinTilesPerCta = 8;  // a CTA gets at least this many key tiles of work
// Work units: a pair's key tiles plus this many units of fixed cost for its
// segment (loading its Q tiles, the epilogue, refilling the pipeline), so that
// a CTA whose range crosses many short pairs is given fewer key tiles.
constexpr int kSegUnits = 2;
// Warps 0-7 softmax, 8 MMA issue, 9-12 K producers, 13-15 V producers. Warpgroups 2-3 (warps 8-15) hand registers to warpgroups 0-1:
// 8 * 32 * kRegSoftmax + 8 * 32 * kRegOther = 512 threads * 128 registers.
constexpr int kThreads = 512;
constexpr int kRegSoftmax = 184;
constexpr int kRegOther = 72;
constexpr int kKWarps = 4;  // producer warps gathering each K tile
constexpr int kVWarps = 3;  // and each V tile
static_assert(8 * 32 * kRegSoftmax + 8 * 32 * kRegOther == kThreads * 128, "register split must match the launch");
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;

template <int D, int BS, int GH>
struct PrefillCfg {
  static constexpr int kTOK = 128 / GH;      // query tokens per Q tile
  static constexpr int kPairTok = 2 * kTOK;  // query tokens per work item
  static constexpr int kHalves = D / 64;     // 128-byte column groups
  static constexpr int kQTileB = 128 * D * 2;
  static constexpr int kKB = kBN * D * 2;    // one K (or V) tile
  // K and V tiles take turns in a ring of slots: K(j) in slot 2j, V(j) in slot
  // 2j + 1 (mod kNSL). A K slot is free again once S(j) is done, a V slot once
  // O += P V(j) is, so the next loads start as early as each allows.
  static constexpr int kNSL = D == 128 ? 4 : 8;
  static constexpr int kBlk = kBN / BS;          // KV blocks per key tile
  static constexpr int kCPR = D / 8;             // 16-byte chunks per key row
  static constexpr int kStageOff = 2 * kQTileB;
  static constexpr int kBarOff = kStageOff + kNSL * kKB;
  // q_full, q_empty, mma_done, kv_full[NSL], kv_empty[NSL], s_full[2], p_full[2], pv_done[2]
  static constexpr int kNumBars = 3 + 2 * kNSL + 6;
  static constexpr int kTmemOff = kBarOff + kNumBars * 8;
  static constexpr int kScanOff = (kTmemOff + 16 + 15) / 16 * 16;
  static constexpr int kSeqOff = kScanOff + 32 * 4;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kOCol = 256;
  static constexpr uint32_t kIdescS = tc::idesc_bf16_f32(128, kBN, 0, 0);
  static constexpr uint32_t kIdescO = tc::idesc_bf16_f32(128, D, 0, 1);
  static size_t smem_bytes(int num_seqs) { return 1024 + kSeqOff + 4ull * (num_seqs + 1); }
};

// 2^x with the hardware's approximate exp2 (denormal results flush to zero,
// 2^-inf = 0): the probabilities are rounded to bf16 right after.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

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
  int adv;           // work units from the segment's start to the next segment
  int64_t tile0;     // unit of the pair's first key tile
};

// The segment of CTA `cta` (unit range [beg, end)) that starts at unit b.
// prefix[s] = work units before sequence s (prefix[num_seqs] > b). A pair of
// nt key tiles occupies kSegUnits + nt units: its fixed cost, then one unit per
// key tile. The segment holds key tiles [j_lo, j_hi) of the pair (possibly none,
// when b and end fall in the fixed-cost units); adv units lead to the next one.
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
  const int units_hg = (prefix[lo + 1] - prefix[lo]) / HGp;
  int off = static_cast<int>(b - prefix[lo]);
  g.hg = off / units_hg;
  off -= g.hg * units_hg;
  int pt = 0, nt;
  int64_t u0 = prefix[lo] + static_cast<int64_t>(g.hg) * units_hg;  // the pair's first unit
  for (;;) {
    nt = tiles_through(g.L, g.ql, min((pt + 1) * PT, g.ql));
    if (off < kSegUnits + nt) break;
    off -= kSegUnits + nt;
    u0 += kSegUnits + nt;
    ++pt;
  }
  g.pt = pt;
  g.nt = nt;
  g.nt0 = tiles_through(g.L, g.ql, min(pt * PT + TOK, g.ql));
  g.t1 = pt * PT + TOK < g.ql;
  g.tile0 = u0 + kSegUnits;
  const int64_t jl = b - g.tile0, jh = end - g.tile0;
  g.j_lo = static_cast<int>(jl > 0 ? jl : 0);
  g.j_hi = static_cast<int>(jh < nt ? (jh > 0 ? jh : 0) : nt);
  const int64_t pair_end = g.tile0 + nt;
  g.adv = static_cast<int>((pair_end < end ? pair_end : end) - b);
  // a split pair's first piece (its tiles start in this CTA) takes slot 2 cta + 1,
  // a later piece (the pair began in an earlier CTA) slot 2 cta
  g.slot = (g.j_lo == 0 && g.j_hi == nt) ? -1 : 2 * cta + (g.j_lo == 0 ? 1 : 0);
}

template <int D, int BS, int GH>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const PrefillArgs a) {
  using C = PrefillCfg<D, BS, GH>;
  constexpr int NSL = C::kNSL;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* mma_done = bars + 2;
  uint64_t* kv_full = bars + 3;     // [NSL]: slot loaded
  uint64_t* kv_empty = kv_full + NSL;  // [NSL]: slot consumed
  uint64_t* s_full = kv_empty + NSL;  // [Q tile]: S computed (and every earlier MMA)
  uint64_t* p_full = s_full + 2;      // [Q tile]: P written (and O rescaled) by its softmax warps
  uint64_t* pv_done = p_full + 2;     // [Q tile]: O += P V done
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
    for (int i = 0; i < NSL; ++i) {
      mbar_init(&kv_full[i], 32 * ((i & 1) ? kVWarps : kKWarps));  // one arrival per lane of the warps that fill it
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp of the Q tile
      mbar_init(&pv_done[i], 1);
    }
    fence_barrier_init();
  }
  if (warp >= kLoadWarp && lane == 0) tma_prefetch_desc(&qmap);
  // The merge grid chained after this one may be scheduled now: its CTAs take
  // SMs as this grid's CTAs exit and wait there for this whole grid to finish,
  // so the merge starts without a launch gap. (The merge grid is launched only
  // once every CTA of this grid has executed this, so none of its CTAs can
  // take an SM that a CTA of this grid still waits for.)
  launch_dependents();

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
          for (int pt = 0; pt * C::kPairTok < ql; ++pt)
            n += kSegUnits + tiles_through(L, ql, min((pt + 1) * C::kPairTok, ql));
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
  // The work item this CTA starts and later CTAs continue, if any: the merge
  // kernel's block for this CTA folds that item's partials together.
  if (tid == 0) {
    int4 rec = make_int4(0, 0, 0, -1);
    if (T > 0 && static_cast<int>(blockIdx.x) < Geff) {
      const int64_t b0 = static_cast<int64_t>(blockIdx.x) * T / Geff;
      const int64_t e0 = static_cast<int64_t>(blockIdx.x + 1) * T / Geff;
      PSeg g;
      locate<GH>(e0 - 1, b0, e0, static_cast<int>(blockIdx.x), prefix, S, HGp, a, g);
      const int64_t ps = g.tile0, pe = g.tile0 + g.nt;  // the item's first and one-past-last key-tile unit
      if (e0 - 1 >= ps && pe > e0 && ps >= b0)
        rec = make_int4(g.r0 + g.pt * C::kPairTok, g.ql - g.pt * C::kPairTok, g.hg * GH, cta_of_block(pe - 1, T, Geff));
    }
    a.pf_split[blockIdx.x] = rec;
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

  // Registers move from warpgroups 2-3 (MMA issue, producers, idle) to the
  // softmax warpgroups: each role calls setmaxnreg first thing.
  if (warp >= kLoadWarp + kKWarps + kVWarps) {
    setmaxnreg_dec<kRegOther>();  // idle warps only hand over their registers
  } else if (warp >= kLoadWarp) {
    setmaxnreg_dec<kRegOther>();
    // ================= producers. kKWarps warps gather every key tile's K and
    // kVWarps its V (so each ring slot is filled by the same warps, in order);
    // warp w of a set takes the tile's rows in groups of 8 (w, w + the set's
    // size, ...), with 16-byte cp.async copies straight into the 128-byte swizzled
    // layout the MMAs read (chunk c of row r at r * 128 + ((c ^ (r & 7)) << 4)
    // within its 64-column half). Rows at or beyond L are filled with zeros, so
    // stale bits in the unfilled tail of the last block never reach the MMAs.
    // Every lane arrives on kv_full asynchronously, when its copies have
    // landed; the MMA thread fences them for the tensor cores. The first K warp
    // also loads each segment's two Q tiles (TMA), after the segment's first K
    // tile (the Q buffer frees only when the previous segment's last scores are
    // done), or before it for the CTA's first segment. (More gathering warps keep more copies in flight: each warp
    // sustains only a few bytes per cycle.)
    const int kv = warp - kLoadWarp < kKWarps ? 0 : 1;          // 0: K, 1: V
    const int wi = kv ? warp - kLoadWarp - kKWarps : warp - kLoadWarp;  // warp within its set
    const int nw = kv ? kVWarps : kKWarps;
    constexpr int RPW = 32 / C::kCPR;                     // rows per warp step
    const int ch = lane % C::kCPR;                        // 16-byte chunk of a row
    const int rl = lane / C::kCPR;                        // row of the step
    const uint32_t dst_col = (ch >> 3) * (kBN * 128);
    const int64_t tok_bytes = static_cast<int64_t>(a.num_kv_heads) * D * 2;
    bool ok = true;
    uint32_t kt = 0, nq = 0;  // key tiles and segments of this CTA so far
    uint32_t my_q = 0;        // 1 + the segment of the last Q load this warp issued (0: none)
    // both Q tiles of segment nq, once the previous segment's scores are done
    auto load_q = [&](const PSeg& g) {
      bool r = true;
      if (lane == 0) {
        r = mbar_wait(q_empty, (nq & 1) ^ 1, a.status, a.wait_limit_ns);
        if (r) {
          mbar_arrive_expect_tx(q_full, 2 * C::kQTileB);
#pragma unroll
          for (int qi = 0; qi < 2; ++qi)
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h)
              tma_load_3d(smem + qi * C::kQTileB + h * 128 * 128, &qmap, q_full, h * 64, g.hg * GH,
                          g.r0 + g.pt * C::kPairTok + qi * C::kTOK);
        }
      }
      r = __shfl_sync(0xffffffffu, r, 0) != 0;
      if (r) my_q = nq + 1;
      return r;
    };
    for (int64_t b = beg; b < end && ok;) {
      PSeg g;
      locate<GH>(b, beg, end, cta, prefix, S, HGp, a, g);
      b += g.adv;
      if (g.j_lo == g.j_hi) continue;  // only fixed-cost units of a pair
      const int hq0 = g.hg * GH, hk = hq0 / G;
      const int* row = a.block_tables + static_cast<size_t>(g.s) * a.max_blocks_per_seq;
      const int nblk_valid = (g.L + BS - 1) / BS;
      const char* src = static_cast<const char*>(kv ? a.v_cache : a.k_cache) + static_cast<size_t>(hk) * D * 2 +
                        ch * 16;
      for (int j = g.j_lo; j < g.j_hi && ok; ++j, ++kt) {
        const int kbase = j * kBN;
        const uint32_t n = 2 * kt + kv, sl = n % NSL;
        if (lane == 0) ok = mbar_wait(&kv_empty[sl], ((n / NSL) & 1) ^ 1, a.status, a.wait_limit_ns);
        ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
        if (!ok) break;
        // the CTA's first Q tiles go out before its first key tile: nothing
        // holds their buffer yet
        if (warp == kLoadWarp && j == g.j_lo && nq == 0) {
          if (!(ok = load_q(g))) break;
        }
        const uint32_t dst = smem_u32(smem + C::kStageOff + sl * C::kKB) + dst_col;
        // the tile's 128 rows in groups of 8 (one block holds whole groups):
        // warp wi takes groups wi, wi + nw, ...
        for (int rgp = wi; rgp < kBN / 8; rgp += nw) {
          const int lb = j * C::kBlk + (rgp * 8) / BS;
          int pb = -1;  // -1: past the sequence (or invalid): the rows are zero-filled
          if (lb < nblk_valid) {
            pb = __ldg(row + lb);
            if (pb < 0 || pb >= a.num_blocks) {
              if (lane == 0 && kv == 1) raise_flag(a.status, PA_FLAG_BLOCK_RANGE);
              pb = -1;
            }
          }
          const char* bsrc = src + (pb >= 0 ? static_cast<int64_t>(pb) * BS * tok_bytes : 0);
#pragma unroll
          for (int i = 0; i < 8 / RPW; ++i) {
            const int r = rgp * 8 + rl + RPW * i;  // row of the tile
            const int t = r % BS;                  // token of the block
            const bool live = pb >= 0 && kbase + r < g.L;
            cp_async16(dst + r * 128 + (((ch & 7) ^ (r & 7)) << 4), bsrc + (live ? t * tok_bytes : 0),
                       live ? 16u : 0u);
          }
        }
        cp_async_arrive(&kv_full[sl]);
        if (warp == kLoadWarp && j == g.j_lo && nq > 0) {  // a later segment's Q tiles
          if (!(ok = load_q(g))) break;
        }
      }
      ++nq;
    }
    // every copy of this thread has landed before the CTA exits
    cp_async_wait_all();
    // the last Q load this warp issued (default bound): one Q load is in flight
    // at a time, since each waits for the previous segment's scores
    if (lane == 0 && my_q > 0) mbar_drain(q_full, (my_q - 1) & 1, a.status);
    __syncwarp();
  } else if (warp == kMmaWarp) {
    setmaxnreg_dec<kRegOther>();
    // ================= MMA issue (lane 0). Per key tile j, for Q tile 0 then 1:
    // O_i += P_i(j-1) V(j-1) once its softmax warps have written P_i(j-1), then
    // S_i(j) = Q_i K(j)^T into the same TMEM columns. The softmax of one Q
    // tile thus runs while the tensor pipe works on the other.
    bool ok = true;
    uint32_t kt = 0, nq = 0;
    uint32_t ns[2] = {0, 0};  // S products issued per Q tile (= P tiles to consume)
    auto wait1 = [&](uint64_t* bar, uint32_t parity) {
      bool r = true;
      if (lane == 0) r = mbar_wait(bar, parity, a.status, a.wait_limit_ns);
      return __shfl_sync(0xffffffffu, r, 0) != 0;
    };
    // O_qi += P_qi V for the V tile in slot sl, whose P is S product number c of Q tile qi
    auto issue_pv = [&](int qi, uint32_t sl, uint32_t c, bool accumulate) {
      if (!wait1(&p_full[qi], c & 1)) return false;
      if (lane == 0) {
        tc::fence_after_sync();
        const uint32_t v_addr = smem_u32(smem + C::kStageOff + sl * C::kKB);
        const uint32_t p_t = tmem + qi * 128;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          tc::mma_bf16_ta(tmem + C::kOCol + qi * D, p_t + kk * 8,
                          tc::sw128_desc(v_addr + kk * 16 * 128, kBN * 128, 1024), C::kIdescO,
                          accumulate || kk > 0);
        tc::commit(&pv_done[qi]);
      }
      return true;
    };
    for (int64_t b = beg; b < end && ok;) {
      PSeg g;
      locate<GH>(b, beg, end, cta, prefix, S, HGp, a, g);
      b += g.adv;
      if (g.j_lo == g.j_hi) continue;  // only fixed-cost units of a pair
      if (!(ok = wait1(q_full, nq & 1))) break;
      ++nq;
      const uint32_t q_addr = smem_u32(smem);
      bool pact[2] = {false, false};     // Q tile active in the previous key tile
      bool acc[2] = {false, false};      // O_i already holds a product of this segment
      uint32_t pc[2] = {0, 0}, pvs = 0;  // its S number, and the previous tile's V slot
      for (int j = g.j_lo; j < g.j_hi; ++j, ++kt) {
        const uint32_t ksl = (2 * kt) % NSL;
        if (!(ok = wait1(&kv_full[ksl], ((2 * kt) / NSL) & 1))) break;
        if (pact[0] || pact[1]) {  // the previous tile's V
          if (!(ok = wait1(&kv_full[pvs], ((2 * kt - 1) / NSL) & 1))) break;
        }
        if (lane == 0) fence_proxy_async_smem();  // the slots were written by cp.async (generic proxy)
        const bool act[2] = {j < g.nt0, g.t1};
        const uint32_t k_addr = smem_u32(smem + C::kStageOff + ksl * C::kKB);
#pragma unroll
        for (int qi = 0; qi < 2; ++qi) {
          if (pact[qi]) {
            if (!(ok = issue_pv(qi, pvs, pc[qi], acc[qi]))) break;
            acc[qi] = true;
          }
          if (act[qi] && lane == 0) {
            const uint32_t qa0 = q_addr + qi * C::kQTileB;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off_q = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
              const uint32_t off_k = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
              tc::mma_bf16(tmem + qi * 128, tc::sw128_desc(qa0 + off_q, 16, 1024),
                           tc::sw128_desc(k_addr + off_k, 16, 1024), C::kIdescS, kk > 0);
            }
            tc::commit(&s_full[qi]);
          }
        }
        if (!ok) break;
        if (lane == 0) {
          tc::commit(&kv_empty[ksl]);                             // K(j) is consumed once S(j) is done
          if (pact[0] || pact[1]) tc::commit(&kv_empty[pvs]);     // V of the previous tile
          if (j == g.j_hi - 1) tc::commit(q_empty);               // every product reading Q is issued
        }
#pragma unroll
        for (int qi = 0; qi < 2; ++qi) {
          pact[qi] = act[qi];
          pc[qi] = ns[qi];
          ns[qi] += act[qi] ? 1 : 0;
        }
        pvs = (2 * kt + 1) % NSL;
      }
      if (!ok) break;
      // the last key tile's products
      if (!(ok = wait1(&kv_full[pvs], ((2 * kt - 1) / NSL) & 1))) break;
      if (lane == 0) fence_proxy_async_smem();
#pragma unroll
      for (int qi = 0; qi < 2; ++qi) {
        if (pact[qi]) {
          if (!(ok = issue_pv(qi, pvs, pc[qi], acc[qi]))) break;
        }
      }
      if (!ok) break;
      if (lane == 0) tc::commit(&kv_empty[pvs]);
    }
    // no MMA may be in flight when TMEM is released
    if (lane == 0) {
      tc::commit(mma_done);
      mbar_drain(mma_done, 0, a.status);
    }
    __syncwarp();
  } else {
    setmaxnreg_inc<kRegSoftmax>();
    // ================= softmax: warps 4 qi .. 4 qi + 3 own Q tile qi, one row per thread
    const int qi = warp >> 2;
    const int r = tid & 127;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_col = qi * 128;
    const uint32_t o_col = C::kOCol + qi * D;
    uint32_t cnt = 0;  // S tiles of this Q tile consumed so far
    bool failed = false;
    for (int64_t b = beg; b < end && !failed;) {
      PSeg g;
      locate<GH>(b, beg, end, cta, prefix, S, HGp, a, g);
      b += g.adv;
      if (g.j_lo == g.j_hi) continue;  // only fixed-cost units of a pair
      const int tok = g.pt * C::kPairTok + qi * C::kTOK + r / GH;
      const int lim = min(g.L - g.ql + tok, g.L - 1);  // last key this row may see
      const int jend = qi == 0 ? min(g.j_hi, g.nt0) : (g.t1 ? g.j_hi : g.j_lo);
      float m_used = -CUDART_INF_F, l = 0.f;
      int done = 0;
      for (int j = g.j_lo; j < jend; ++j) {
        failed = !mbar_wait(&s_full[qi], cnt & 1, a.status, a.wait_limit_ns);
        if (__any_sync(0xffffffffu, failed)) {
          failed = true;
          break;
        }
        tc::fence_after_sync();
        float sv[kBN];
#pragma unroll
        for (int q = 0; q < kBN / 32; ++q) tc::ld32(t_lane + s_col + 32 * q, sv + 32 * q);
        tc::wait_ld();
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
        l *= alpha;
        // a row that sees no key of this segment yet keeps m = -inf: its
        // probabilities are exactly 0 (exp2 of -inf)
        const float m_e = m_used == -CUDART_INF_F ? 0.f : m_used;
        // P over the first 64 columns of this tile's S (already in registers)
        float2 lq = make_float2(0.f, 0.f);
        const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-m_e, -m_e);
#pragma unroll
        for (int q = 0; q < kBN / 32; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 x = __ffma2_rn(make_float2(sv[32 * q + 2 * i], sv[32 * q + 2 * i + 1]), sc2, nm2);
            const float2 e = make_float2(ex2_ftz(x.x), ex2_ftz(x.y));
            lq = __fadd2_rn(lq, e);
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(e.x, e.y);
            pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          tc::st16u(t_lane + s_col + 16 * q, pk);
        }
        l += lq.x + lq.y;
        // O holds every product up to the previous tile (a completed S implies
        // the earlier P.V completed): rescale it before this tile's product
        if (j > g.j_lo && __any_sync(0xffffffffu, bump)) {
#pragma unroll 1
          for (int q = 0; q < D / 32; ++q) {
            float ov[32];
            tc::ld32(t_lane + o_col + 32 * q, ov);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            tc::st32(t_lane + o_col + 32 * q, ov);
          }
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[qi]);
        ++cnt;
        ++done;
      }
      if (failed) break;
      if (done > 0) {
        // the segment's last product of this Q tile is number cnt - 1
        failed = !mbar_wait(&pv_done[qi], (cnt - 1) & 1, a.status, a.wait_limit_ns);
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
              // fp16 (11-bit significand, |O / l| <= max |V|): its rounding stays
              // well under the bf16 rounding of the merged row. Layout
              // [slot][column / 8][256 rows][8]: a warp's 32 rows of one 8-column
              // group are 512 contiguous bytes, so each store is coalesced.
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4) {
                uint16_t* po = a.pf_o + ((static_cast<size_t>(g.slot) * (D / 8) + 4 * q + v4) * 256 + qi * 128 + r) * 8;
                uint32_t pk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const __half2 h2 = __floats2half2_rn(ov[8 * v4 + 2 * i] * inv_l, ov[8 * v4 + 2 * i + 1] * inv_l);
                  pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                *reinterpret_cast<uint4*>(po) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              }
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
// that CTA x starts and CTAs x + 1 .. continue (its split record); blockIdx.y
// selects 32 of its 256 rows; a warp's lanes are 32 consecutive rows of one
// group of D / 8 columns (so each partial load is 512 contiguous bytes).
// O = sum_k 2^(lse_k - M) O_k / sum_k 2^(lse_k - M).
template <int D, int GH>
__global__ void __launch_bounds__(256) prefill_combine_kernel(const PrefillArgs a) {
  constexpr int TOK = 128 / GH, kCols = D / 8;
  grid_dependency_wait();  // the prefill grid (partials and split records) is complete
  const int c = blockIdx.x;
  const int4 rec = a.pf_split[c];  // first query row of the pair, rows left, first head, last CTA
  if (rec.w < 0) return;
  const int row = blockIdx.y * 32 + (threadIdx.x & 31);
  const int qi = row >> 7, rr = row & 127;
  const int tok = qi * TOK + rr / GH;
  if (tok >= rec.y) return;
  const int col0 = (threadIdx.x >> 5) * kCols;
  const int np = rec.w - c + 1;  // pieces: this CTA's (slot 2c + 1), then slot 2cc of CTA cc
  auto slot_of = [&](int k) { return k == 0 ? 2 * c + 1 : 2 * (c + k); };
  float M = -CUDART_INF_F, sum = 0.f, acc[kCols];
#pragma unroll
  for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
  // O += w f, skipping a piece no key of which reaches the row (its O was not written)
  auto fold = [&](float lse, const uint4* u) {
    if (lse == -CUDART_INF_F) return;
    const float w = fast_exp2(lse - M);
    sum += w;
#pragma unroll
    for (int i = 0; i < kCols / 8; ++i) {
      const uint32_t w4[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[k]));
        acc[8 * i + 2 * k] = fmaf(w, f.x, acc[8 * i + 2 * k]);
        acc[8 * i + 2 * k + 1] = fmaf(w, f.y, acc[8 * i + 2 * k + 1]);
      }
    }
  };
  auto load_row = [&](int slot, uint4* u) {
#pragma unroll
    for (int i = 0; i < kCols / 8; ++i)
      u[i] = *reinterpret_cast<const uint4*>(a.pf_o + ((static_cast<size_t>(slot) * (D / 8) + col0 / 8 + i) * 256 + row) * 8);
  };
  constexpr int kMaxP = 4;
  if (np <= kMaxP) {
    // every load of the thread issued at once (a row not written is loaded but never used)
    float lse[kMaxP];
    uint4 u[kMaxP][kCols / 8];
#pragma unroll
    for (int k = 0; k < kMaxP; ++k) {
      lse[k] = -CUDART_INF_F;
      if (k < np) {
        lse[k] = a.pf_lse[static_cast<size_t>(slot_of(k)) * 256 + row];
        load_row(slot_of(k), u[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < kMaxP; ++k) M = fmaxf(M, lse[k]);
#pragma unroll
    for (int k = 0; k < kMaxP; ++k) fold(lse[k], u[k]);
  } else {
    for (int k = 0; k < np; ++k) M = fmaxf(M, a.pf_lse[static_cast<size_t>(slot_of(k)) * 256 + row]);
    for (int k = 0; k < np; ++k) {
      uint4 u[kCols / 8];
      load_row(slot_of(k), u);
      fold(a.pf_lse[static_cast<size_t>(slot_of(k)) * 256 + row], u);
    }
  }
  const float inv = 1.f / sum;
  __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) +
                        (static_cast<size_t>(rec.x + tok) * a.num_q_heads + rec.z + rr % GH) * D + col0;
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
  const int64_t tiles = pairs * (kSegUnits + (static_cast<int64_t>(max_context_len) + kBN - 1) / kBN);
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
