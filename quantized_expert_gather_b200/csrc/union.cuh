// Route-union on one warp: the distinct experts of a window in ascending order,
// each expert's (token, expert) pairs in ascending pair id, and the offsets.
//
// "Small-L fused expert gather for fine-grained MoE decode" (mlx discussion
// 3801), second post: sort the (position, expert) pairs by expert, stream each
// unique expert once, apply it to the ragged set of positions routed to it.
//
// Method (stable counting sort with warp primitives):
//   1. pairs are taken 32 at a time in ascending order; __match_any_sync groups
//      the lanes holding the same expert, so a pair's rank among the earlier
//      pairs of its expert is the running count plus the number of lower
//      lanes in its group; the group's lowest lane bumps the count;
//   2. one pass over the experts turns the counts into the ascending list of
//      used experts (__ballot_sync + __popc prefix) and into start offsets
//      (warp inclusive scan);
//   3. each pair lands at start[e] + rank.
// Pair ids outside [0, E) are left out and raise kErrExpertIndex.
#pragma once

#include "common.cuh"

namespace qeg {

struct UnionView {
  int u;                 // number of distinct valid experts
  int n_valid;           // number of valid pairs (= offsets[u])
  const int* unique;     // [u]
  const int* offsets;    // [u + 1]
  const int* pair_list;  // [n_valid]
};

// Run by all 32 lanes of one warp.  Arrays may live in shared or global
// memory; `cnt` needs E ints and `rank` P ints of scratch.  On return (after
// the warp's own __syncwarp) the outputs are written; the caller makes them
// visible to other warps.  pair_list entries past n_valid are set to -1.
// Returns u; *n_valid_out receives the number of valid pairs.
__device__ inline int warp_route_union(const int* __restrict__ idx, int P, int E, int* cnt,
                                       int* rank, int* unique, int* offsets, int* pair_list,
                                       int* n_valid_out) {
  const int lane = threadIdx.x & 31;
  if (P <= 32) {
    // A window of at most 32 pairs: one key (expert, pair) per lane, sorted across the
    // warp by a bitonic network (15 compare-exchange steps), so no pass over the E
    // experts is needed.  Invalid pairs sort last and are left out.
    const int e = lane < P ? idx[lane] : -1;
    const bool valid = lane < P && e >= 0 && e < E;
    if (__any_sync(kFull, lane < P && !valid)) {
      if (lane == 0) set_error(kErrExpertIndex);
    }
    int key = valid ? ((e << 5) | lane) : 0x7fffffff;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        const int other = __shfl_xor_sync(kFull, key, j);
        const bool keep_min = ((lane & j) == 0) == ((lane & k) == 0);
        key = keep_min ? min(key, other) : max(key, other);
      }
    const bool kv = key != 0x7fffffff;
    const int ke = key >> 5;
    const int prev = __shfl_up_sync(kFull, ke, 1);
    const bool first = kv && (lane == 0 || prev != ke);
    const unsigned heads = __ballot_sync(kFull, first);
    const int nv = __popc(__ballot_sync(kFull, kv));
    if (first) {
      const int slot = __popc(heads & lanemask_lt());
      unique[slot] = ke;
      offsets[slot] = lane;
    }
    const int u = __popc(heads);
    if (lane == 0) offsets[u] = nv;
    if (lane < P) pair_list[lane] = kv ? (key & 31) : -1;
    __syncwarp();
    *n_valid_out = nv;
    return u;
  }
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  bool bad = false;
  for (int base = 0; base < P; base += 32) {
    const int p = base + lane;
    const int e = (p < P) ? idx[p] : -1;
    const bool valid = (p < P) && e >= 0 && e < E;
    bad |= (p < P) && !valid;
    const int key = valid ? e : -1 - lane;  // invalid lanes match nobody
    const unsigned grp = __match_any_sync(kFull, key);
    const int old = valid ? cnt[e] : 0;
    __syncwarp();
    if (valid && lane == __ffs(grp) - 1) cnt[e] = old + __popc(grp);
    if (p < P) rank[p] = valid ? old + __popc(grp & lanemask_lt()) : -1;
    __syncwarp();
  }
  if (__any_sync(kFull, bad)) {
    if (lane == 0) set_error(kErrExpertIndex);
  }
  int u = 0, off = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const int c = (e < E) ? cnt[e] : 0;
    const unsigned used = __ballot_sync(kFull, c > 0);
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, d);
      if (lane >= d) incl += v;
    }
    if (c > 0) {
      const int slot = u + __popc(used & lanemask_lt());
      unique[slot] = e;
      offsets[slot] = off + incl - c;
      cnt[e] = off + incl - c;  // start offset of expert e
    }
    u += __popc(used);
    off += __shfl_sync(kFull, incl, 31);
  }
  __syncwarp();
  if (lane == 0) offsets[u] = off;
  for (int p = lane; p < P; p += 32) {
    const int r = rank[p];
    if (r >= 0) pair_list[cnt[idx[p]] + r] = p;
  }
  for (int i = off + lane; i < P; i += 32) pair_list[i] = -1;
  __syncwarp();
  *n_valid_out = off;
  return u;
}

}  // namespace qeg
