// Router step ahead of the layer: for every token, the k experts with the largest
// logits (descending; the lower expert id first among equal logits) and their
// softmax probabilities, renormalised over the k picks (or left over all E).  This
// is how the tiny parity configuration routes its tokens (top-k of softmax,
// renormalised over the k); the output feeds moe_switchglu_forward directly.
//
// One warp per token.  The row is staged in shared memory; k rounds of a warp-wide
// arg-max over (logit, then lower id) pick the experts, lane j keeping the j-th
// pick.  A probability is exp(l - m), m the row's largest logit, divided by the sum
// over the picks (renormalised) or over the whole row.  Logits must be finite.
#pragma once

#include <cmath>

#include "common.cuh"

namespace qeg {

constexpr int kRouterWarps = 8;      // tokens per CTA
constexpr int kRouterMaxE = 1024;    // experts (the library's limit)
constexpr int kRouterMaxK = 32;      // picks per token: one lane each

// One token's picks by one warp: the row `row` (E logits, global) is staged in v / taken
// (E floats and E bytes of this warp's scratch); lane j < k returns the j-th pick in
// *idx (-1 if none) and its probability in *w.  Run by all 32 lanes.
__device__ __forceinline__ void router_row(const float* __restrict__ row, int E, int k,
                                           int renormalize, float* v, unsigned char* taken,
                                           int lane, int* idx, float* w) {
  for (int e = lane; e < E; e += 32) {
    v[e] = __ldg(row + e);
    taken[e] = 0;
  }
  __syncwarp();

  float my_val = 0.f, m = 0.f;
  int my_idx = -1;
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float x = v[e];
      if (!taken[e] && (x > bv || (x == bv && e < bi))) {
        bv = x;
        bi = e;
      }
    }
    // arg-max over the warp: a total order, so every lane ends with the same pick
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, off);
      const int oi = __shfl_xor_sync(kFull, bi, off);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    const bool valid = bi < E;  // always, for finite logits
    if (r == 0) m = bv;
    if (lane == r) {
      my_val = bv;
      my_idx = valid ? bi : -1;
    }
    if (lane == 0 && valid) taken[bi] = 1;
    __syncwarp();
  }

  const float ex = (lane < k && my_idx >= 0) ? expf(my_val - m) : 0.f;
  float denom = 0.f;
  if (renormalize) {
    denom = ex;
  } else {
    for (int e = lane; e < E; e += 32) denom += expf(v[e] - m);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) denom += __shfl_xor_sync(kFull, denom, off);
  *idx = my_idx;
  *w = ex / denom;
  __syncwarp();  // v and taken may be reused for the next row
}

__global__ void __launch_bounds__(32 * kRouterWarps)
    router_topk_kernel(const float* __restrict__ logits, int T, int E, int k, int renormalize,
                       int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  __shared__ float s_val[kRouterWarps][kRouterMaxE];
  __shared__ unsigned char s_taken[kRouterWarps][kRouterMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouterWarps + warp;
  if (t >= T) return;  // warp-uniform
  int pi;
  float pw;
  router_row(logits + (size_t)t * E, E, k, renormalize, s_val[warp], s_taken[warp], lane, &pi,
             &pw);
  if (lane < k) {
    topk_idx[(size_t)t * k + lane] = pi;
    topk_w[(size_t)t * k + lane] = pw;
  }
}

}  // namespace qeg
