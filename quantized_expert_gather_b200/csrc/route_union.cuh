// Standalone route-union kernel (one CTA of 32 warps) for any pair count.
//
// Same output as warp_route_union (union.cuh): the distinct routed experts in
// ascending order, offsets, and the pairs grouped by expert in ascending pair
// id.  Stable counting sort over 32 warps, each owning a contiguous slice of
// the pairs:
//   1. per-warp histograms hist[w][e] built with __match_any_sync;
//   2. per expert, an exclusive prefix over the warps (the slice order keeps
//      the sort stable) and the expert's total;
//   3. one warp turns the totals into unique[] and offsets[] (ballot + scan),
//      and optionally padded[], the same prefix over counts rounded up to 16
//      (the row offsets of the grouped kernels' packed activation layout);
//   4. each warp re-walks its slice and places every pair at
//      offsets[slot(e)] + (pairs of e in earlier slices) + (earlier pairs of e
//      in this slice).
#pragma once

#include "common.cuh"

namespace qeg {

constexpr int kUnionWarps = 32;

__host__ __device__ inline size_t route_union_smem_bytes(int E) {
  return sizeof(int) * ((size_t)kUnionWarps * E + 2 * (size_t)E) + 64;
}

__global__ void __launch_bounds__(32 * kUnionWarps, 1)
    route_union_kernel(const int* __restrict__ idx, int P, int E, int* __restrict__ unique,
                       int* __restrict__ offsets, int* __restrict__ pair_list,
                       int* __restrict__ num_unique, int* __restrict__ padded = nullptr) {
  extern __shared__ __align__(16) int su[];
  int* hist = su;                        // [kUnionWarps][E]
  int* total = su + kUnionWarps * E;     // [E]
  int* base = total + E;                 // [E]  start offset of expert e
  __shared__ int s_valid;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (P + kUnionWarps - 1) / kUnionWarps;
  const int p_begin = min(P, warp * per), p_end = min(P, p_begin + per);

  for (int i = threadIdx.x; i < kUnionWarps * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();

  // 1. histograms
  int* h = hist + warp * E;
  bool bad = false;
  for (int b = p_begin; b < p_end; b += 32) {
    const int p = b + lane;
    const int e = (p < p_end) ? idx[p] : -1;
    const bool valid = (p < p_end) && e >= 0 && e < E;
    bad |= (p < p_end) && !valid;
    const unsigned grp = __match_any_sync(kFull, valid ? e : -1 - lane);
    if (valid && lane == __ffs(grp) - 1) h[e] += __popc(grp);
    __syncwarp();
  }
  if (__any_sync(kFull, bad) && lane == 0) set_error(kErrExpertIndex);
  __syncthreads();

  // 2. prefix over warps, per expert
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kUnionWarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    total[e] = run;
  }
  __syncthreads();

  // 3. unique experts and offsets
  if (warp == 0) {
    int u = 0, off = 0, poff = 0;
    for (int b = 0; b < E; b += 32) {
      const int e = b + lane;
      const int c = (e < E) ? total[e] : 0;
      const int pc = (c + 15) & ~15;  // the expert's pairs rounded up to 16
      const unsigned used = __ballot_sync(kFull, c > 0);
      int incl = c, pincl = pc;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, d);
        const int pv = __shfl_up_sync(kFull, pincl, d);
        if (lane >= d) {
          incl += v;
          pincl += pv;
        }
      }
      if (c > 0) {
        const int slot = u + __popc(used & lanemask_lt());
        unique[slot] = e;
        offsets[slot] = off + incl - c;
        base[e] = off + incl - c;
        if (padded != nullptr) padded[slot] = poff + pincl - pc;
      }
      u += __popc(used);
      off += __shfl_sync(kFull, incl, 31);
      poff += __shfl_sync(kFull, pincl, 31);
    }
    if (lane == 0) {
      offsets[u] = off;
      if (padded != nullptr) padded[u] = poff;
      *num_unique = u;
      s_valid = off;
    }
  }
  __syncthreads();

  // 4. placement
  for (int b = p_begin; b < p_end; b += 32) {
    const int p = b + lane;
    const int e = (p < p_end) ? idx[p] : -1;
    const bool valid = (p < p_end) && e >= 0 && e < E;
    const unsigned grp = __match_any_sync(kFull, valid ? e : -1 - lane);
    const int before = valid ? h[e] : 0;
    __syncwarp();
    if (valid) {
      pair_list[base[e] + before + __popc(grp & lanemask_lt())] = p;
      if (lane == __ffs(grp) - 1) h[e] = before + __popc(grp);
    }
    __syncwarp();
  }
  for (int i = s_valid + threadIdx.x; i < P; i += blockDim.x) pair_list[i] = -1;
}

}  // namespace qeg
