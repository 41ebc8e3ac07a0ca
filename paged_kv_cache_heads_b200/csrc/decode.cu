// Paged decode attention (query rows with q_len == 1), split-K over the block
// table with an online softmax, plus the kernel that merges the splits.
//
// What is computed: for sequence s with L = context_lens[s] keys and query
// head h, o = softmax(q . K[0:L]^T * scale) . V[0:L], where key i lives in
// row i % bs of physical block block_tables[s][i / bs] for KV head
// h / (Hq / Hkv). The logical-to-physical walk is the page table of
// "vLLM核心架构：PagedAttention原理、KV Cache管理、连续批处理机制",
// §"一、PagedAttention：虚拟内存的灵感"; the decode call is the one the page
// "深入解析 nano-vLLM 推理引擎的分页 KV 缓存与内存优化架构",
// §"工程落地：配置参数与监控指标" hands to a library; that page (§三 of the
// first) notes decode is bound by memory bandwidth, which shapes this design.
//
// Design (B200):
//  * Work item = (sequence, group of GH query heads sharing one KV head,
//    split of the sequence's keys). Splits of one sequence are equal-sized
//    multiples of the block size, so items are balanced.
//  * Persistent CTAs (a multiple of the SM count) walk items round-robin.
//    One producer warp gathers each KV block of the item's KV head with two
//    TMA tensor loads (K, V: box {D, 1, bs, 1}) into a ring of NST shared
//    memory stages; the ring keeps running across items, so the HBM stream
//    never drains between items.
//  * NCW consumer warps take the ring's blocks round-robin. Within a warp,
//    LPR lanes hold one 16-byte slice each of a key row (TPW rows per warp
//    step); q.k is a 16-byte-vector dot product finished with a butterfly
//    shuffle. Each warp keeps its own running max m, sum l and fp32
//    accumulator; the warps merge through shared memory at the end of an item.
//  * GQA: every KV block is read once for the GH query heads of the group.
//  * Keys at or beyond L (the unfilled tail of the last block) are masked and
//    their V rows are never read, so stale bits there (even NaN) cannot leak.
//  * A sequence with one split writes its output rows directly; otherwise
//    each split writes (o / l, m + log2 l) to the workspace and a second
//    kernel merges them: O = sum_j 2^(lse_j - M) O_j / sum_j 2^(lse_j - M).
#include <math_constants.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

// Number of equal splits for a sequence of L keys, and their span (a multiple
// of the block size, at most chunk tokens).
__device__ __forceinline__ int split_span(int L, int chunk, int bs) {
  const int n0 = (L + chunk - 1) / chunk;
  const int per = (L + n0 - 1) / n0;
  return ((per + bs - 1) / bs) * bs;
}
__device__ __forceinline__ int num_splits(int L, int chunk, int bs) {
  const int span = split_span(L, chunk, bs);
  return (L + span - 1) / span;
}

// Block-wide inclusive scan of one int per thread (nthreads <= 1024).
__device__ __forceinline__ int block_inclusive_scan(int x, int* warp_tot, int& total) {
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

template <typename T, int D, int BS, int GH, int NCW>
struct DecodeCfg {
  static constexpr int kEB = sizeof(T);
  static constexpr int kRowB = D * kEB;             // bytes of one key row (one head)
  static constexpr int kLPR = kRowB / 16;           // lanes per row
  static constexpr int kTPW = 32 / kLPR;            // rows per warp step
  static constexpr int kEPL = 16 / kEB;             // elements per lane
  static constexpr int kSteps = BS / kTPW;          // warp steps per block
  static constexpr int kNIT = kSteps < 8 ? kSteps : 8;  // steps per softmax update
  static constexpr int kNUPD = kSteps / kNIT;
  static constexpr int kStageB = 2 * BS * kRowB;    // K block + V block
  // Stages: about 64 KiB in flight, and a multiple of NCW so that every use of
  // a stage belongs to the same consumer warp (its parity waits then never
  // run more than one phase ahead of the barrier).
  static constexpr int kNST0 = 65536 / kStageB;
  static constexpr int kNST1 = kNST0 < NCW ? NCW : (kNST0 > 16 ? 16 : kNST0);
  static constexpr int kNST = (kNST1 / NCW) * NCW;
  static constexpr int kThreads = (NCW + 1) * 32;
  static constexpr int kCombFloats = NCW * GH * (D + 2);
  // dynamic smem: stages | bars | comb x2 | warp totals | prefix, clen, row
  static constexpr int kBarOff = kNST * kStageB;
  static constexpr int kCombOff = kBarOff + 2 * kNST * 8;
  static constexpr int kScanOff = kCombOff + 2 * kCombFloats * 4;
  static constexpr int kAbortOff = kScanOff + 32 * 4;
  static constexpr int kSeqOff = kAbortOff + 16;
  static_assert(kRowB % 16 == 0 && 32 % kLPR == 0, "row must split into lanes");
  static_assert(BS % kTPW == 0 && kSteps % kNIT == 0, "block must split into steps");
  static_assert(kNST % NCW == 0, "each stage must always go to the same consumer warp");
  static size_t smem_bytes(int num_seqs) { return 1024 + kSeqOff + 12ull * (num_seqs + 1); }
};

template <typename T, int D, int BS, int GH, int NCW>
__global__ void __launch_bounds__((NCW + 1) * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const DecodeArgs a) {
  using C = DecodeCfg<T, D, BS, GH, NCW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + C::kNST;
  float* comb = reinterpret_cast<float*>(smem + C::kCombOff);
  int* warp_tot = reinterpret_cast<int*>(smem + C::kScanOff);
  volatile int* abort_word = reinterpret_cast<volatile int*>(smem + C::kAbortOff);
  int* prefix = reinterpret_cast<int*>(smem + C::kSeqOff);      // [S+1]
  int* clen = prefix + (a.num_seqs + 1);                         // [S]
  int* qrow = clen + a.num_seqs;                                 // [S]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.num_q_heads / a.num_kv_heads;
  const int HG = a.num_q_heads / GH;  // head groups over all KV heads
  const int chunk = a.chunk_tokens;

  if (tid == 0) {
    for (int i = 0; i < C::kNST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    fence_barrier_init();
    *abort_word = 0;
  }
  if (warp == NCW && lane == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  // The split merge (and any prefill grid) may be scheduled now; the merge
  // waits for this grid's completion before it reads a partial.
  launch_dependents();

  // ---- enumerate the work items of every sequence (decode rows only)
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
        if (L < 1 || L > a.max_context_len || L > a.max_blocks_per_seq * BS) {
          raise_flag(a.status, PA_FLAG_CONTEXT_RANGE);
        } else {
          n = num_splits(L, chunk, BS) * HG;
        }
      }
    }
    int total;
    const int incl = block_inclusive_scan(n, warp_tot, total);
    if (s < a.num_seqs) prefix[s + 1] = carry + incl;
    carry += total;
  }
  __syncthreads();
  const int W = prefix[a.num_seqs];

  // item -> (sequence, split, head group, key-block range)
  auto decode_item = [&](int w, int& s, int& j, int& hg, int& blo, int& bhi, int& L) {
    int lo = 0, hi = a.num_seqs;  // find s: prefix[s] <= w < prefix[s+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= w) lo = mid; else hi = mid;
    }
    s = lo;
    const int r = w - prefix[s];
    j = r / HG;
    hg = r - j * HG;
    L = clen[s];
    const int span = split_span(L, chunk, BS);
    const int t0 = j * span;
    const int t1 = min(t0 + span, L);
    blo = t0 / BS;
    bhi = (t1 + BS - 1) / BS;
  };

  if (warp == NCW) {
    // ================= producer warp: TMA gathers of K/V blocks
    uint32_t k = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < W && ok; w += gridDim.x) {
      int s, j, hg, blo, bhi, L;
      decode_item(w, s, j, hg, blo, bhi, L);
      const int hk = (hg * GH) / G;
      const int* row = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq;
      for (int b0 = blo; b0 < bhi && ok; b0 += 32) {
        int phys = -1;
        if (b0 + lane < bhi) {
          phys = __ldg(row + b0 + lane);
          if (phys < 0 || phys >= a.num_blocks) {
            raise_flag(a.status, PA_FLAG_BLOCK_RANGE);
            phys = -1;  // a fully out-of-bounds box: TMA fills zeros, reads nothing
          }
        }
        const int cnt = min(32, bhi - b0);
        for (int i = 0; i < cnt; ++i, ++k) {
          const int pb = __shfl_sync(0xffffffffu, phys, i);
          int good = 1;
          if (lane == 0) {
            const uint32_t st = k % C::kNST, use = k / C::kNST;
            good = mbar_wait(&empty[st], (use & 1) ^ 1, a.status);
            if (good) {
              uint8_t* dst = smem + st * C::kStageB;
              mbar_arrive_expect_tx(&full[st], C::kStageB);
              tma_load_4d(dst, &kmap, &full[st], 0, hk, 0, pb);
              tma_load_4d(dst + BS * C::kRowB, &vmap, &full[st], 0, hk, 0, pb);
            }
          }
          ok = __shfl_sync(0xffffffffu, good, 0) != 0;
          if (!ok) break;
        }
      }
    }
    return;
  }

  // ================= consumer warps
  const int sub = lane / C::kLPR;  // which row of a warp step
  const int c = lane % C::kLPR;    // which 16-byte slice of the row
  uint32_t k = 0;
  int item_no = 0;
  for (int w = blockIdx.x; w < W; w += gridDim.x, ++item_no) {
    int s, j, hg, blo, bhi, L;
    decode_item(w, s, j, hg, blo, bhi, L);
    const int nblk = bhi - blo;
    const int h0 = hg * GH;
    const int row = qrow[s];

    float qf[GH][C::kEPL];
#pragma unroll
    for (int g = 0; g < GH; ++g) {
      const uint4 qv = *reinterpret_cast<const uint4*>(
          static_cast<const uint8_t*>(a.q) +
          ((static_cast<size_t>(row) * a.num_q_heads + h0 + g) * D + c * C::kEPL) * C::kEB);
      Elem<T>::widen(qv, qf[g]);
#pragma unroll
      for (int e = 0; e < C::kEPL; ++e) qf[g][e] *= a.scale_log2;
    }
    float m[GH], l[GH], acc[GH][C::kEPL];
#pragma unroll
    for (int g = 0; g < GH; ++g) {
      m[g] = -CUDART_INF_F;
      l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < C::kEPL; ++e) acc[g][e] = 0.f;
    }

    bool ok = true;
    const int first = (warp - static_cast<int>(k % NCW) + NCW) % NCW;
    for (int i = first; i < nblk; i += NCW) {
      const uint32_t kk = k + i;
      const uint32_t st = kk % C::kNST;
      if (!mbar_wait(&full[st], (kk / C::kNST) & 1, a.status)) { ok = false; break; }
      const uint8_t* Ks = smem + st * C::kStageB;
      const uint8_t* Vs = Ks + BS * C::kRowB;
      const int tok0 = (blo + i) * BS;
#pragma unroll
      for (int u = 0; u < C::kNUPD; ++u) {
        float sc[GH][C::kNIT];
#pragma unroll
        for (int it = 0; it < C::kNIT; ++it) {
          const int t = (u * C::kNIT + it) * C::kTPW + sub;
          const uint4 kv = *reinterpret_cast<const uint4*>(Ks + t * C::kRowB + c * 16);
          float kf[C::kEPL];
          Elem<T>::widen(kv, kf);
#pragma unroll
          for (int g = 0; g < GH; ++g) {
            float p = 0.f;
#pragma unroll
            for (int e = 0; e < C::kEPL; ++e) p = fmaf(qf[g][e], kf[e], p);
            sc[g][it] = p;
          }
        }
#pragma unroll
        for (int it = 0; it < C::kNIT; ++it) {
          const bool valid = tok0 + (u * C::kNIT + it) * C::kTPW + sub < L;
#pragma unroll
          for (int g = 0; g < GH; ++g) {
            float p = sc[g][it];
#pragma unroll
            for (int off = C::kLPR / 2; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
            sc[g][it] = valid ? p : -CUDART_INF_F;
          }
        }
#pragma unroll
        for (int g = 0; g < GH; ++g) {
          float mx = sc[g][0];
#pragma unroll
          for (int it = 1; it < C::kNIT; ++it) mx = fmaxf(mx, sc[g][it]);
#pragma unroll
          for (int off = C::kLPR; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          const float m_new = fmaxf(m[g], mx);
          const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
          const float alpha = fast_exp2(m[g] - m_use);
          m[g] = m_new;
          l[g] *= alpha;
#pragma unroll
          for (int e = 0; e < C::kEPL; ++e) acc[g][e] *= alpha;
#pragma unroll
          for (int it = 0; it < C::kNIT; ++it) {
            const float p = fast_exp2(sc[g][it] - m_use);
            sc[g][it] = p;
            l[g] += p;
          }
        }
#pragma unroll
        for (int it = 0; it < C::kNIT; ++it) {
          const int t = (u * C::kNIT + it) * C::kTPW + sub;
          if (tok0 + t < L) {
            const uint4 vv = *reinterpret_cast<const uint4*>(Vs + t * C::kRowB + c * 16);
            float vf[C::kEPL];
            Elem<T>::widen(vv, vf);
#pragma unroll
            for (int g = 0; g < GH; ++g)
#pragma unroll
              for (int e = 0; e < C::kEPL; ++e) acc[g][e] = fmaf(sc[g][it], vf[e], acc[g][e]);
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
    for (int g = 0; g < GH; ++g) {
#pragma unroll
      for (int off = C::kLPR; off < 32; off <<= 1) {
        l[g] += __shfl_xor_sync(0xffffffffu, l[g], off);
#pragma unroll
        for (int e = 0; e < C::kEPL; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], off);
      }
    }
    float* cb = comb + (item_no & 1) * C::kCombFloats + warp * GH * (D + 2);
    if (sub == 0) {
#pragma unroll
      for (int g = 0; g < GH; ++g) {
#pragma unroll
        for (int e = 0; e < C::kEPL; ++e) cb[g * (D + 2) + c * C::kEPL + e] = acc[g][e];
        if (c == 0) {
          cb[g * (D + 2) + D] = m[g];
          cb[g * (D + 2) + D + 1] = l[g];
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
    if (*abort_word) return;  // every consumer warp sees the same value here

    // ---- merge the warps; write the output row or this split's partial
    const float* cball = comb + (item_no & 1) * C::kCombFloats;
    const int nsplit = num_splits(L, chunk, BS);
    for (int idx = tid; idx < GH * D; idx += NCW * 32) {
      const int g = idx / D, d = idx - g * D;
      float M = -CUDART_INF_F;
#pragma unroll
      for (int ww = 0; ww < NCW; ++ww) M = fmaxf(M, cball[(ww * GH + g) * (D + 2) + D]);
      float sl = 0.f, so = 0.f;
#pragma unroll
      for (int ww = 0; ww < NCW; ++ww) {
        const float* pw = cball + (ww * GH + g) * (D + 2);
        const float f = fast_exp2(pw[D] - M);
        sl = fmaf(pw[D + 1], f, sl);
        so = fmaf(pw[d], f, so);
      }
      const float o = so / sl;
      if (nsplit == 1) {
        static_cast<T*>(a.out)[(static_cast<size_t>(row) * a.num_q_heads + h0 + g) * D + d] = Elem<T>::narrow(o);
      } else {
        const size_t part = (static_cast<size_t>(s) * a.max_splits + j) * a.num_q_heads + h0 + g;
        a.part_o[part * D + d] = o;
        if (d == 0) a.part_lse[part] = M + log2f(sl);
      }
    }
  }
}

// One CTA per (sequence, query head): merge the splits of a decode row.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeArgs a) {
  launch_dependents();
  grid_dependency_wait();  // every partial of the decode grid is written
  const int s = blockIdx.x / a.num_q_heads;
  const int h = blockIdx.x - s * a.num_q_heads;
  const int r0 = __ldg(a.query_start_loc + s);
  if (__ldg(a.query_start_loc + s + 1) - r0 != 1) return;
  const int L = __ldg(a.context_lens + s);
  if (L < 1 || L > a.max_context_len || L > a.max_blocks_per_seq * BS) return;
  const int n = num_splits(L, a.chunk_tokens, BS);
  if (n <= 1) return;
  const size_t base = static_cast<size_t>(s) * a.max_splits * a.num_q_heads + h;
  float M = -CUDART_INF_F;
  for (int j = 0; j < n; ++j) M = fmaxf(M, a.part_lse[base + static_cast<size_t>(j) * a.num_q_heads]);
  float sw = 0.f, so = 0.f;
  const int d = threadIdx.x;
  for (int j = 0; j < n; ++j) {
    const size_t p = base + static_cast<size_t>(j) * a.num_q_heads;
    const float w = fast_exp2(a.part_lse[p] - M);
    sw += w;
    so = fmaf(w, a.part_o[p * D + d], so);
  }
  static_cast<T*>(a.out)[(static_cast<size_t>(r0) * a.num_q_heads + h) * D + d] = Elem<T>::narrow(so / sw);
}

constexpr int kNCW = 4;

template <typename T, int D, int BS, int GH>
cudaError_t launch_decode_t(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            cudaStream_t stream) {
  using C = DecodeCfg<T, D, BS, GH, kNCW>;
  auto kern = paged_decode_kernel<T, D, BS, GH, kNCW>;
  const size_t smem = C::smem_bytes(a.num_seqs);
  static int configured_smem[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && configured_smem[dev] < static_cast<int>(smem)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured_smem[dev] = static_cast<int>(smem);
  }
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t items_bound =
      static_cast<int64_t>(a.num_seqs) * (a.num_q_heads / GH) * a.max_splits;
  const int64_t slots = static_cast<int64_t>(num_sms()) * per_sm;
  const int grid = static_cast<int>(items_bound < slots ? (items_bound > 0 ? items_bound : 1) : slots);
  kern<<<grid, C::kThreads, smem, stream>>>(kmap, vmap, a);
  return cudaGetLastError();
}

template <typename T, int D, int BS>
cudaError_t launch_decode_gh(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                             cudaStream_t stream) {
  switch (decode_heads_per_cta(a.num_q_heads / a.num_kv_heads)) {
    case 4: return launch_decode_t<T, D, BS, 4>(a, kmap, vmap, stream);
    case 2: return launch_decode_t<T, D, BS, 2>(a, kmap, vmap, stream);
    default: return launch_decode_t<T, D, BS, 1>(a, kmap, vmap, stream);
  }
}

template <typename T, int D>
cudaError_t launch_decode_bs(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                             int bs, cudaStream_t stream) {
  switch (bs) {
    case 8: return launch_decode_gh<T, D, 8>(a, kmap, vmap, stream);
    case 16: return launch_decode_gh<T, D, 16>(a, kmap, vmap, stream);
    default: return launch_decode_gh<T, D, 32>(a, kmap, vmap, stream);
  }
}

template <typename T, int D>
cudaError_t launch_combine_bs(const DecodeArgs& a, int bs, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(a.num_seqs) * a.num_q_heads;
  switch (bs) {
    case 8: return launch_chained(decode_combine_kernel<T, D, 8>, dim3(grid), dim3(D), 0, stream, a);
    case 16: return launch_chained(decode_combine_kernel<T, D, 16>, dim3(grid), dim3(D), 0, stream, a);
    default: return launch_chained(decode_combine_kernel<T, D, 32>, dim3(grid), dim3(D), 0, stream, a);
  }
}

}  // namespace

int32_t decode_heads_per_cta(int32_t group) {
  if (group % 4 == 0) return 4;
  if (group % 2 == 0) return 2;
  return 1;
}

cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          const pa_cache_desc& c, cudaStream_t stream) {
  if (c.dtype == PA_BF16) {
    if (c.head_dim == 64) return launch_decode_bs<__nv_bfloat16, 64>(a, kmap, vmap, c.block_size, stream);
    return launch_decode_bs<__nv_bfloat16, 128>(a, kmap, vmap, c.block_size, stream);
  }
  if (c.head_dim == 64) return launch_decode_bs<float, 64>(a, kmap, vmap, c.block_size, stream);
  return launch_decode_bs<float, 128>(a, kmap, vmap, c.block_size, stream);
}

cudaError_t launch_decode_combine(const DecodeArgs& a, const pa_cache_desc& c, cudaStream_t stream) {
  if (c.dtype == PA_BF16) {
    if (c.head_dim == 64) return launch_combine_bs<__nv_bfloat16, 64>(a, c.block_size, stream);
    return launch_combine_bs<__nv_bfloat16, 128>(a, c.block_size, stream);
  }
  if (c.head_dim == 64) return launch_combine_bs<float, 64>(a, c.block_size, stream);
  return launch_combine_bs<float, 128>(a, c.block_size, stream);
}

int32_t decode_chunk_tokens(int32_t num_seqs, int32_t num_kv_heads, int32_t group,
                            int32_t max_context_len, int32_t block_size) {
  // Aim for several items per resident CTA slot so the round-robin tail is
  // short, assuming the average sequence is half the longest one; never split
  // finer than 4 blocks or coarser than 512 tokens.
  const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads *
                        (group / decode_heads_per_cta(group));
  const int64_t target_items = 8ll * 148 * 2;
  const int64_t avg_tokens = max_context_len > 1 ? max_context_len / 2 : 1;
  int64_t chunk = units > 0 ? (units * avg_tokens + target_items - 1) / target_items : 512;
  const int64_t lo = 4ll * block_size;
  if (chunk < lo) chunk = lo;
  if (chunk > 512) chunk = 512;
  chunk = ((chunk + block_size - 1) / block_size) * block_size;
  if (const char* env = getenv("PA_DECODE_CHUNK")) {
    const int64_t v = atoll(env);
    if (v >= block_size) chunk = (v / block_size) * block_size;
  }
  return static_cast<int32_t>(chunk);
}

}  // namespace pa
