// Work partition shared by the decode kernels (CUDA-core and tensor-core).
//
// A unit is (sequence, group of query heads read from one KV head). Its work
// is the sequence's ceil(L/bs) KV blocks. All units' blocks are numbered
// contiguously, unit-major; a persistent grid of G CTAs splits that range
// evenly, CTA c taking blocks [c*B/G, (c+1)*B/G). The part of one unit that
// one CTA streams is a segment. A unit that one CTA covers entirely is written
// straight to the output; otherwise each covering CTA c writes partial slot
// u + c (unique: the CTAs covering unit u+1 start where those of unit u end)
// and the merge kernel combines them.
#pragma once

#include <stdint.h>

namespace pa {

// First CTA whose range [c*B/G, (c+1)*B/G) contains block b (0 <= b < B).
__device__ __forceinline__ int cta_of_block(int64_t b, int64_t B, int G) {
  return static_cast<int>(((b + 1) * G - 1) / B);
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

// One segment: the part of a unit's block range that one CTA streams.
struct Segment {
  int s;         // sequence
  int hg;        // head group (first query head hg * heads-per-unit)
  int blo, bhi;  // logical blocks [blo, bhi) of the sequence
  int L;         // context length (filled by the caller)
  int slot;      // partial slot (unit + cta), or -1 when this CTA covers the whole unit
  int skip;      // leading table blocks left to the cascade prefix pass (0 without cascade)
};

// The segment of CTA `cta`, whose range is [beg, end), that starts at global
// block b (beg <= b < end). prefix[s] = decode blocks of sequences before s;
// HG = units per sequence.
__device__ __forceinline__ void locate_segment(int64_t b, const int* prefix, int num_seqs, int HG, int64_t beg,
                                               int64_t end, int cta, Segment& g) {
  int lo = 0, hi = num_seqs;  // largest s with prefix[s] * HG <= b
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<int64_t>(prefix[mid]) * HG <= b) lo = mid; else hi = mid;
  }
  const int nbs = prefix[lo + 1] - prefix[lo];
  const int64_t off = b - static_cast<int64_t>(prefix[lo]) * HG;
  const int hg = static_cast<int>(off / nbs);
  const int lb = static_cast<int>(off - static_cast<int64_t>(hg) * nbs);
  const int64_t ub0 = b - lb, ub1 = ub0 + nbs;  // the unit's global block range
  g.s = lo;
  g.hg = hg;
  g.blo = lb;
  g.bhi = lb + static_cast<int>(nbs - lb < end - b ? nbs - lb : end - b);
  g.slot = (ub0 >= beg && ub1 <= end) ? -1 : (lo * HG + hg) + cta;
  g.skip = 0;
}

// Cascade decode: a sequence whose first `skip` blocks the prefix pass reads
// streams only blocks [skip, ...) and always leaves a partial for the merge.
__device__ __forceinline__ void apply_skip(const int32_t* skip_blocks, int HG, int cta, Segment& g) {
  if (!skip_blocks) return;
  g.skip = __ldg(skip_blocks + g.s);
  if (g.skip > 0 && g.slot < 0) g.slot = (g.s * HG + g.hg) + cta;
}

}  // namespace pa
