// The union-of-experts SwitchGLU layer as one persistent kernel (one CTA per
// SM), for small token windows (T*k <= kMaxPairsFused).
//
// "Small-L fused expert gather for fine-grained MoE decode" (mlx discussion
// 3801, first post, "Two implications" item 1): compute the union of routed
// experts across the window, stream each selected expert's weights once, and
// apply them to whichever positions routed to it.
//
//   prologue  route-union of the window (every CTA forms the same union in
//             shared memory from topk_idx), cut into segments: an expert and up
//             to `seg` of its pairs;
//   phase A   gate+up over blocks (segment, kRowsA rows of Wg and Wu):
//               h = bf16(silu(bf16(Wg x)) * bf16(Wu x))
//             (the one-pass epilogue of "Apple7/8 MoE gate and up in one decode
//             pass", splash PR 45, "What changed"), h stored per pair;
//   phase B   down over blocks (segment, rows_b rows of Wd): y = Wd h per pair,
//             stored fp32.  A segment's phase-B blocks start once every phase-A
//             block of that segment has published its h (counter hdone[seg]);
//   combine   out[t] = bf16(sum_j w[t,j] * y[t,j]), j ascending, per block of
//             rows_b output rows, run by the CTA that completes the last segment
//             of that row block (counter ydone[rb]) -- no grid-wide barrier.
// Blocks are split evenly over the CTAs.  An expert with more than `seg` pairs
// in the window forms several segments and is streamed once per segment.
// Every spin on a counter is bounded (common.cuh); the CTA that finishes last
// resets the counters, so the workspace counters are zero between calls.
//
// Memory pipeline: a ring of kStages shared-memory stages fed by 1-D bulk
// copies (cp.async.bulk, mbarrier completion) runs through phases A and B as
// one sequence of blocks, so the first phase-B blocks stream while phase A
// finishes.  Every warp computes; the last warp to finish a stage (shared-memory
// counter) issues the copy kStages blocks ahead.
//
// Compute: each warp owns whole rows (phase A: one row of Wg and the same row
// of Wu; phase B: up to 4 rows of Wd) over the full input width.  Lane l takes
// the 32-column chunks l, l+32, ... of its rows, so one lane chunk sits inside
// one quantisation group (64 columns):
//     partial = s * sum_c q_c x_c + b * sum_c x_c.
// The segment's activations sit in shared memory as 16-bit block fixed point
// (one exponent per 32-column chunk, see below), so that sum_c q_c x_c is an
// exact integer dot product of the 4-bit codes with the activation's two bytes
// (dp4a), scaled once per chunk.  A warp reduces its rows over its lanes once per
// block; there is no cross-warp exchange inside a phase.
#pragma once

#include "common.cuh"
#include "union.cuh"

namespace qeg {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRowsA = kWarps;      // phase A: one row of gate and of up per warp per block
constexpr int kMaxRowsPerWarpB = 4; // phase B: rows of Wd per warp per block
constexpr int kStages = 4;          // ring depth
constexpr int kNT = 4;              // pairs per segment (upper bound)
constexpr int kMaxPairsFused = 1024;
constexpr unsigned kXBytes = 64 * 1024;  // activation buffer (block fixed point)

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------- geometry ---
struct LayerGeom {
  int rounds_a, rounds_b;  // 32-column chunks per lane per row (power of two >= H/1024, I/1024)
  int rows_b;              // phase B rows per block (multiple of kWarps, <= 32)
  int seg;                 // pairs per segment (<= kNT)
  unsigned a_q, a_sb, a_mat, a_bytes;  // phase A block: per matrix codes / scale bytes
  unsigned b_q, b_sb, b_bytes;         // phase B full block
  unsigned stage_bytes;
};

__host__ __device__ inline LayerGeom layer_geom(int H, int I) {
  LayerGeom g;
  g.rounds_a = 1;
  while (g.rounds_a * 1024 < H) g.rounds_a <<= 1;
  g.rounds_b = 1;
  while (g.rounds_b * 1024 < I) g.rounds_b <<= 1;
  int rb = (16 * H / I) / kWarps * kWarps;  // about one phase-A stage worth of Wd rows
  if (rb < kWarps) rb = kWarps;
  if (rb > kWarps * kMaxRowsPerWarpB) rb = kWarps * kMaxRowsPerWarpB;
  g.rows_b = rb;
  const int rmax = g.rounds_a > g.rounds_b ? g.rounds_a : g.rounds_b;
  int s = (int)(kXBytes / (2048u * (unsigned)rmax));  // fixed point: rounds * 2 KB per pair
  g.seg = s > kNT ? kNT : s;
  g.a_q = kRowsA * H / 2;
  g.a_sb = kRowsA * H / 32;
  g.a_mat = g.a_q + 2 * g.a_sb;
  g.a_bytes = 2 * g.a_mat;
  g.b_q = g.rows_b * I / 2;
  g.b_sb = g.rows_b * I / 32;
  g.b_bytes = g.b_q + 2 * g.b_sb;
  g.stage_bytes = (unsigned)align_up(g.a_bytes > g.b_bytes ? g.a_bytes : g.b_bytes, 128);
  return g;
}

struct LayerSmem {
  size_t stages, x, xsum, cnt, rank, unique, offsets, pair_list, pos_of, seg_slot, seg_pos,
      seg_nt, comb, total;
};
__host__ __device__ inline LayerSmem layer_smem(const LayerGeom& g, int E, int P, int H, int I) {
  LayerSmem s;
  const int m = (E < P ? E : P) > 0 ? (E < P ? E : P) : 1;
  const int rmax = g.rounds_a > g.rounds_b ? g.rounds_a : g.rounds_b;
  s.stages = 0;
  s.x = align_up((size_t)kStages * g.stage_bytes, 128);
  s.xsum = s.x + kXBytes;
  s.cnt = align_up(s.xsum + sizeof(float2) * kNT * rmax * 32, 16);
  s.rank = align_up(s.cnt + sizeof(int) * E, 16);
  s.unique = align_up(s.rank + sizeof(int) * P, 16);
  s.offsets = align_up(s.unique + sizeof(int) * m, 16);
  s.pair_list = align_up(s.offsets + sizeof(int) * (m + 1), 16);
  s.pos_of = align_up(s.pair_list + sizeof(int) * P, 16);
  // segments: at most P of them
  s.seg_slot = align_up(s.pos_of + sizeof(int) * P, 16);
  s.seg_pos = align_up(s.seg_slot + sizeof(int) * P, 16);
  s.seg_nt = align_up(s.seg_pos + sizeof(int) * P, 16);
  s.comb = align_up(s.seg_nt + sizeof(int) * P, 16);  // row blocks to combine (<= rows / 8)
  s.total = align_up(s.comb + sizeof(int) * (H / kWarps + 1), 16);
  return s;
}

// Workspace counters (unsigned), a region of fixed size at the start of every
// workspace so that calls of different shapes never see each other's data there:
// [0] CTAs finished, [1, 1+kMaxPairsFused) hdone per segment, then ydone per
// phase-B row block (at most kMaxRowBlocks).
constexpr int kMaxRowBlocks = 4096 / kWarps;
constexpr size_t kSyncWords = 1 + kMaxPairsFused + kMaxRowBlocks;

// -------------------------------------------------------------- arguments ---
struct LayerArgs {
  const uint16_t* x;  // [T, H] bf16
  const int* idx;     // [T, k]
  const float* w;     // [T, k]
  const uint32_t *gq, *uq, *dq;
  const uint16_t *gs, *gb, *us, *ub, *ds, *db;
  uint16_t* h;        // workspace [P, I] bf16, rows in pair_list order
  float* y;           // workspace [P, H] fp32, rows in pair_list order
  unsigned* sync;     // workspace counters: [0] exit count, [1..] hdone[P], then ydone[]
  int *ex_u, *ex_unique, *ex_offsets, *ex_pair_list;  // union export (CTA 0), may be null
  uint16_t* out;      // [T, H] bf16
  int T, k, E, H, I;
  LayerGeom g;
  int wait_prior;     // wait for the preceding grid before reading any input
};

// ------------------------------------------------- activations and codes ---
// A segment's activations (x rows in phase A, h rows in phase B) are held in
// shared memory as 16-bit block fixed point, one block per 32-column chunk:
//   x_c = v_c * 2^(e - 14),  v_c an integer in [-32640, 32640],
// where e is the exponent of the block's largest magnitude.  A bf16 value whose
// exponent is within 7 of e is held exactly (8 significant bits); smaller ones are
// rounded to the nearest multiple of 2^(e - 14), an error below 2^-15 of the
// block's largest magnitude.  v_c is split into a low byte (unsigned) and a high
// byte (signed), so that a chunk's sum  sum_c q_c v_c  is formed exactly in
// integers by dp4a over 4-bit codes: the codes of a 32-bit word w are split into
// qa = w & 0x0F0F0F0F (columns 0, 2, 4, 6 of the word, one per byte) and
// qb = (w >> 4) & 0x0F0F0F0F (columns 1, 3, 5, 7).
//
// Layout: token t, chunk ch = i * 32 + l (l = lane, i < R): uint4
// xq[((t * R + i) * 4 + m) * 32 + l] covers columns 32 ch + 8m .. +7 as
//   .x = low bytes of columns 8m+0,2,4,6   .y = low bytes of 8m+1,3,5,7
//   .z = high bytes of columns 8m+0,2,4,6  .w = high bytes of 8m+1,3,5,7
// and float2 xsc[t * R * 32 + ch] = (2^(e - 14), sum of the chunk's 32 values).
constexpr uint32_t kNibbleBytes = 0x0F0F0F0Fu;

__device__ __forceinline__ int dp4a_lo(uint32_t q, uint32_t d, int c) {
  return static_cast<int>(__dp4a(q, d, static_cast<unsigned>(c)));
}
__device__ __forceinline__ int dp4a_hi(uint32_t q, uint32_t d, int c) {
  return __dp4a(static_cast<int>(q), static_cast<int>(d), c);
}

// A chunk's activation quarters (token t, round i) into registers.
__device__ __forceinline__ void load_xq(const uint4* xq, int t, int R, int i, int lane,
                                        uint4 (&d)[4]) {
  const uint4* p = xq + ((size_t)(t * R + i) * 4) * 32 + lane;
#pragma unroll
  for (int m = 0; m < 4; ++m) d[m] = p[m * 32];
}

// sum_c q_c v_c over one chunk (4 code words, 4 activation uint4), exact.
__device__ __forceinline__ int chunk_dot(const uint32_t (&qs)[8], const uint4 (&x)[4]) {
  int lo = 0, hi = 0;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint4 d = x[m];
    lo = dp4a_lo(qs[2 * m], d.x, lo);
    lo = dp4a_lo(qs[2 * m + 1], d.y, lo);
    hi = dp4a_hi(qs[2 * m], d.z, hi);
    hi = dp4a_hi(qs[2 * m + 1], d.w, hi);
  }
  return hi * 256 + lo;  // |.| < 2^24: exact in fp32
}

// The 32 codes of a uint4, split as described above.
__device__ __forceinline__ void split_codes(const uint4 v, uint32_t (&qs)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    qs[2 * m] = w[m] & kNibbleBytes;
    qs[2 * m + 1] = (w[m] >> 4) & kNibbleBytes;
  }
}

// One thread's quarter of a chunk: the 8 bf16 values of columns 8m .. 8m+7 (in v)
// become this thread's uint4 of the layout above; the 4 threads of a chunk are
// consecutive lanes (group mask gmask).  Returns the chunk's (scale, sum) in every
// thread of the group.
__device__ __forceinline__ float2 fixed_point_quarter(const uint4 v, unsigned gmask,
                                                      uint4& out) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  int X[8], M[8], neg[8];
  int xm = 0;
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t b = (k & 1) ? (w[k >> 1] >> 16) : (w[k >> 1] & 0xffffu);
    const int ex = (b >> 7) & 0xff, mant = b & 0x7f;
    M[k] = ex ? (mant | 0x80) : mant;
    X[k] = ex ? ex : 1;
    neg[k] = (b >> 15) & 1;
    if (M[k]) xm = max(xm, X[k]);
    sum += __uint_as_float(b << 16);
  }
  xm = max(xm, __shfl_xor_sync(gmask, xm, 1, 4));
  xm = max(xm, __shfl_xor_sync(gmask, xm, 2, 4));
  sum += __shfl_xor_sync(gmask, sum, 1, 4);
  sum += __shfl_xor_sync(gmask, sum, 2, 4);
  uint32_t lo[2] = {0u, 0u}, hi[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int sh = xm - X[k];  // >= 0 for every nonzero value
    int mag;
    if (sh <= 7) mag = M[k] << (7 - sh);
    else if (sh <= 15) mag = (M[k] + (1 << (sh - 8))) >> (sh - 7);  // round half up
    else mag = 0;
    const int val = neg[k] ? -mag : mag;
    const int pos = (k >> 1) * 8;  // byte within the word; k even -> .x/.z, odd -> .y/.w
    lo[k & 1] |= (static_cast<uint32_t>(val) & 0xffu) << pos;
    hi[k & 1] |= ((static_cast<uint32_t>(val) >> 8) & 0xffu) << pos;
  }
  out = make_uint4(lo[0], lo[1], hi[0], hi[1]);
  float scale;
  if (xm == 0) scale = 0.f;                                    // all zero
  else if (xm == 255) scale = __uint_as_float(0x7fc00000u);   // Inf / NaN present
  else if (xm >= 15) scale = __uint_as_float(static_cast<uint32_t>(xm - 14) << 23);
  else scale = __uint_as_float(1u << (xm + 8));               // 2^(xm-141), subnormal
  return make_float2(scale, sum);
}

// ---------------------------------------------------------------- counters ---
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_gpu(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Spin (bounded) until *p >= target.  Returns false and sets kErrTimeout if the
// limit runs out.
__device__ __forceinline__ bool wait_counter(const unsigned* p, unsigned target) {
  if (ld_acquire_gpu(p) >= target) return true;
  const unsigned long long t0 = globaltimer();
  while (ld_acquire_gpu(p) < target) {
    __nanosleep(32);
    if (globaltimer() - t0 > kWaitLimitNs) {
      set_error(kErrTimeout);
      return false;
    }
  }
  return true;
}

// --------------------------------------------------------- per-warp compute ---
// Phase A: this warp's row of Wg and of Wu, NT pairs, R rounds of 32-column chunks
// (chunks past H/32 skipped); returns (G, U) for t < NT in every lane.  Per chunk
// (inside one quantisation group): s * 2^(e-14) * sum q v + b * sum x.
template <int NT, int R>
__device__ __forceinline__ void rows_a(const unsigned char* bg_q, const uint16_t* bg_s,
                                       const uint16_t* bg_b, const unsigned char* bu_q,
                                       const uint16_t* bu_s, const uint16_t* bu_b, int H,
                                       const uint4* xq, const float2* xsc, int lane,
                                       float (&G)[kNT], float (&U)[kNT]) {
  float ag[NT], au[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) ag[t] = au[t] = 0.f;
  const int nch = H / 32;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int ch = i * 32 + lane;
    if (ch < nch) {
      uint32_t qg[8], qu[8];
      split_codes(*reinterpret_cast<const uint4*>(bg_q + ch * 16), qg);
      split_codes(*reinterpret_cast<const uint4*>(bu_q + ch * 16), qu);
      const float sg = bf16_bits_to_float(bg_s[ch >> 1]), bgv = bf16_bits_to_float(bg_b[ch >> 1]);
      const float su = bf16_bits_to_float(bu_s[ch >> 1]), buv = bf16_bits_to_float(bu_b[ch >> 1]);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        uint4 xd[4];
        load_xq(xq, t, R, i, lane, xd);
        const float2 sc = xsc[t * R * 32 + ch];
        const float dg = static_cast<float>(chunk_dot(qg, xd));
        const float du = static_cast<float>(chunk_dot(qu, xd));
        ag[t] = fmaf(sg * sc.x, dg, fmaf(bgv, sc.y, ag[t]));
        au[t] = fmaf(su * sc.x, du, fmaf(buv, sc.y, au[t]));
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
      ag[t] += __shfl_xor_sync(kFull, ag[t], m);
      au[t] += __shfl_xor_sync(kFull, au[t], m);
    }
    G[t] = ag[t];
    U[t] = au[t];
  }
}

// Phase B: rows row0 + kWarps*q (q < kMaxRowsPerWarpB, rows < nrows) of Wd, NT pairs.
// Returns the value this lane holds after a reduce-scatter and its index
// q*kNT + t in `vid` (-1 when it holds none).
template <int NT, int R>
__device__ __forceinline__ float rows_b(const unsigned char* bq, const uint16_t* bs,
                                        const uint16_t* bb, int row0, int nrows, int I,
                                        const uint4* xq, const float2* xsc, int lane, int& vid) {
  constexpr int NP = (NT == 3) ? 4 : NT;
  constexpr int V = kMaxRowsPerWarpB * NP;
  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  const int nch = I / 32, qstride = I / 2, sstride = I / 64;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int ch = i * 32 + lane;
    if (ch < nch) {
      float2 sc[NT];
      uint4 xd[NT][4];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        sc[t] = xsc[t * R * 32 + ch];
        load_xq(xq, t, R, i, lane, xd[t]);
      }
#pragma unroll
      for (int q = 0; q < kMaxRowsPerWarpB; ++q) {
        const int r = row0 + kWarps * q;
        if (r < nrows) {
          uint32_t qs[8];
          split_codes(*reinterpret_cast<const uint4*>(bq + (size_t)r * qstride + ch * 16), qs);
          const float sv = bf16_bits_to_float(bs[r * sstride + (ch >> 1)]);
          const float bv = bf16_bits_to_float(bb[r * sstride + (ch >> 1)]);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float d = static_cast<float>(chunk_dot(qs, xd[t]));
            acc[q * NP + t] = fmaf(sv * sc[t].x, d, fmaf(bv, sc[t].y, acc[q * NP + t]));
          }
        }
      }
    }
  }
  int v_id;
  const float v = warp_reduce_scatter<V>(acc, lane, v_id);
  constexpr int kHolderMask = (32 / V) - 1;
  const int q = v_id / NP, t = v_id % NP;
  vid = ((lane & kHolderMask) == 0 && t < NT) ? q * kNT + t : -1;
  return v;
}

// ------------------------------------------------------------------ kernel ---
template <int NT>
__device__ __forceinline__ void dispatch_a(int R, const unsigned char* bgq, const uint16_t* bgs,
                                           const uint16_t* bgb, const unsigned char* buq,
                                           const uint16_t* bus, const uint16_t* bub, int H,
                                           const uint4* xq, const float2* xsc, int lane,
                                           float (&G)[kNT], float (&U)[kNT]) {
  if (R == 1) rows_a<NT, 1>(bgq, bgs, bgb, buq, bus, bub, H, xq, xsc, lane, G, U);
  else if (R == 2) rows_a<NT, 2>(bgq, bgs, bgb, buq, bus, bub, H, xq, xsc, lane, G, U);
  else rows_a<NT, 4>(bgq, bgs, bgb, buq, bus, bub, H, xq, xsc, lane, G, U);
}

template <int NT>
__device__ __forceinline__ float dispatch_b(int R, const unsigned char* bq, const uint16_t* bs,
                                            const uint16_t* bb, int row0, int nrows, int I,
                                            const uint4* xq, const float2* xsc, int lane,
                                            int& vid) {
  if (R == 1) return rows_b<NT, 1>(bq, bs, bb, row0, nrows, I, xq, xsc, lane, vid);
  if (R == 2) return rows_b<NT, 2>(bq, bs, bb, row0, nrows, I, xq, xsc, lane, vid);
  if (R == 4) return rows_b<NT, 4>(bq, bs, bb, row0, nrows, I, xq, xsc, lane, vid);
  return rows_b<NT, 8>(bq, bs, bb, row0, nrows, I, xq, xsc, lane, vid);
}

// Estimated time of one block, in units of about 100 SM cycles: the larger of the
// time its bytes take at the SM's share of HBM bandwidth and the time its dequant
// work takes with nt pairs (measured on B200 for the 4096 / 2048 layer).
__device__ __forceinline__ unsigned block_cost_a(int nt) { return max(16, 8 + 7 * nt); }
__device__ __forceinline__ unsigned block_cost_b(int nt) { return max(16, 13 + 6 * nt); }

// Index of the block at which the cumulative cost reaches `target` in a
// segment-major block list (bpe blocks per segment, prefix sums pre[0..nseg]).
// Monotone in target, 0 at 0 and nseg * bpe at the total, so consecutive targets
// cut the list into contiguous, disjoint ranges.
__device__ inline int cost_to_block(const unsigned* pre, const int* seg_nt, int nseg, int bpe,
                                    bool phase_b, unsigned target) {
  if (nseg == 0 || target >= pre[nseg]) return nseg * bpe;
  int lo = 0, hi = nseg;  // largest s with pre[s] <= target, s < nseg
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pre[mid] <= target) lo = mid;
    else hi = mid;
  }
  const unsigned per = phase_b ? block_cost_b(seg_nt[lo]) : block_cost_a(seg_nt[lo]);
  const int r = (int)min((unsigned)bpe, (target - pre[lo]) / per);
  return lo * bpe + r;
}

__global__ void __launch_bounds__(kThreads, 1) layer_kernel(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_u, s_nseg, s_ncomb, s_part[4];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ int stage_cnt[kStages];
  const LayerGeom& G = a.g;
  const int P = a.T * a.k;
  const LayerSmem L = layer_smem(G, a.E, P, a.H, a.I);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned* exit_cnt = a.sync;
  unsigned* hdone = a.sync + 1;
  unsigned* ydone = a.sync + 1 + kMaxPairsFused;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      stage_cnt[s] = 0;
    }
    fence_barrier_init();
  }
  if (a.wait_prior) grid_dep_wait();

  // ---- route-union (warp 0), its segments, and the inverse map pair -> position ----
  int* uniq = reinterpret_cast<int*>(smem + L.unique);
  int* offs = reinterpret_cast<int*>(smem + L.offsets);
  int* plist = reinterpret_cast<int*>(smem + L.pair_list);
  int* pos_of = reinterpret_cast<int*>(smem + L.pos_of);
  int* seg_slot = reinterpret_cast<int*>(smem + L.seg_slot);
  int* seg_pos = reinterpret_cast<int*>(smem + L.seg_pos);
  int* seg_nt = reinterpret_cast<int*>(smem + L.seg_nt);
  int* comb = reinterpret_cast<int*>(smem + L.comb);
  if (warp == 0) {
    int nv;
    const int u = warp_route_union(a.idx, P, a.E, reinterpret_cast<int*>(smem + L.cnt),
                                   reinterpret_cast<int*>(smem + L.rank), uniq, offs, plist, &nv);
    // segments: expert slot i contributes ceil(n_i / seg) segments, in slot order
    int base = 0;
    for (int b0 = 0; b0 < u; b0 += 32) {
      const int i = b0 + lane;
      const int n_i = (i < u) ? offs[i + 1] - offs[i] : 0;
      const int c = (n_i + G.seg - 1) / G.seg;
      int incl = c;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += v;
      }
      for (int j = 0; j < c; ++j) {
        const int s = base + incl - c + j;
        seg_slot[s] = i;
        seg_pos[s] = offs[i] + j * G.seg;
        seg_nt[s] = min(G.seg, n_i - j * G.seg);
      }
      base += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) {
      s_u = u;
      s_nseg = base;
    }
  } else {
    for (int p = threadIdx.x - 32; p < P; p += kThreads - 32) pos_of[p] = -1;
  }
  __syncthreads();
  const int u = s_u, nseg = s_nseg;
  const int n_valid = offs[u];
  for (int i = threadIdx.x; i < n_valid; i += kThreads) pos_of[plist[i]] = i;

  // ---- this CTA's blocks: phase A [a0, a0+na), phase B [b0, b0+nb) ----
  // Each phase's block list (segment-major) is cut into equal shares of estimated
  // cost, so that CTAs holding segments with more pairs get fewer blocks.  The
  // prefix sums live in the stage buffers, which no copy has touched yet.
  const int bpe_a = a.I / kRowsA;
  const int bpe_b = (a.H + G.rows_b - 1) / G.rows_b;
  unsigned* pre_a = reinterpret_cast<unsigned*>(smem + L.stages);
  unsigned* pre_b = pre_a + (nseg + 1);
  if (warp == 0) {
    unsigned run_a = 0, run_b = 0;
    for (int c0 = 0; c0 < nseg; c0 += 32) {
      const int sgi = c0 + lane;
      unsigned ca = 0, cb = 0;
      if (sgi < nseg) {
        ca = block_cost_a(seg_nt[sgi]) * (unsigned)bpe_a;
        cb = block_cost_b(seg_nt[sgi]) * (unsigned)bpe_b;
      }
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const unsigned va = __shfl_up_sync(kFull, ca, d), vb = __shfl_up_sync(kFull, cb, d);
        if (lane >= d) {
          ca += va;
          cb += vb;
        }
      }
      if (sgi < nseg) {
        pre_a[sgi + 1] = run_a + ca;
        pre_b[sgi + 1] = run_b + cb;
      }
      run_a += __shfl_sync(kFull, ca, 31);
      run_b += __shfl_sync(kFull, cb, 31);
    }
    if (lane == 0) pre_a[0] = pre_b[0] = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned G_ = gridDim.x, c = blockIdx.x;
    const unsigned long long ta = pre_a[nseg], tb = pre_b[nseg];
    const int x0 = cost_to_block(pre_a, seg_nt, nseg, bpe_a, false, (unsigned)(ta * c / G_));
    const int x1 = cost_to_block(pre_a, seg_nt, nseg, bpe_a, false, (unsigned)(ta * (c + 1) / G_));
    const int y0 = cost_to_block(pre_b, seg_nt, nseg, bpe_b, true, (unsigned)(tb * c / G_));
    const int y1 = cost_to_block(pre_b, seg_nt, nseg, bpe_b, true, (unsigned)(tb * (c + 1) / G_));
    s_part[0] = x0;
    s_part[1] = x1 - x0;
    s_part[2] = y0;
    s_part[3] = y1 - y0;
  }
  __syncthreads();
  const int a0 = s_part[0], na = s_part[1], b0 = s_part[2], nb = s_part[3];
  const int ng = na + nb;

  // copy block g of this CTA's sequence into stage g % kStages (one thread)
  auto issue = [&](int gi) {
    const int st = gi % kStages;
    unsigned char* buf = smem + L.stages + (size_t)st * G.stage_bytes;
    if (gi < na) {
      const int blk = a0 + gi, sg = blk / bpe_a, row0 = (blk % bpe_a) * kRowsA;
      const size_t r0 = (size_t)uniq[seg_slot[sg]] * a.I + row0;
      const size_t qrow = a.H / 8, srow = a.H / 64;
      mbar_arrive_expect_tx(&full[st], G.a_bytes);
      bulk_g2s(buf, a.gq + r0 * qrow, G.a_q, &full[st]);
      bulk_g2s(buf + G.a_q, a.gs + r0 * srow, G.a_sb, &full[st]);
      bulk_g2s(buf + G.a_q + G.a_sb, a.gb + r0 * srow, G.a_sb, &full[st]);
      buf += G.a_mat;
      bulk_g2s(buf, a.uq + r0 * qrow, G.a_q, &full[st]);
      bulk_g2s(buf + G.a_q, a.us + r0 * srow, G.a_sb, &full[st]);
      bulk_g2s(buf + G.a_q + G.a_sb, a.ub + r0 * srow, G.a_sb, &full[st]);
    } else {
      const int blk = b0 + (gi - na), sg = blk / bpe_b, row0 = (blk % bpe_b) * G.rows_b;
      const int nrows = min(G.rows_b, a.H - row0);
      const size_t r0 = (size_t)uniq[seg_slot[sg]] * a.H + row0;
      const size_t qrow = a.I / 8, srow = a.I / 64;
      const unsigned qb = nrows * (a.I / 2), sb = nrows * (a.I / 32);
      mbar_arrive_expect_tx(&full[st], qb + 2 * sb);
      bulk_g2s(buf, a.dq + r0 * qrow, qb, &full[st]);
      bulk_g2s(buf + G.b_q, a.ds + r0 * srow, sb, &full[st]);
      bulk_g2s(buf + G.b_q + G.b_sb, a.db + r0 * srow, sb, &full[st]);
    }
  };
  if (threadIdx.x == 0) {
    fence_proxy_async();  // the stage buffers held the prefix sums (generic writes)
    for (int gi = 0; gi < ng && gi < kStages; ++gi) issue(gi);
  }

  if (blockIdx.x == 0 && warp == 1 && a.ex_u) {
    for (int i = lane; i < u; i += 32) a.ex_unique[i] = uniq[i];
    for (int i = lane; i <= u; i += 32) a.ex_offsets[i] = offs[i];
    for (int i = lane; i < P; i += 32) a.ex_pair_list[i] = plist[i];
    if (lane == 0) *a.ex_u = u;
  }

  uint4* xq = reinterpret_cast<uint4*>(smem + L.x);
  float2* xsc = reinterpret_cast<float2*>(smem + L.xsum);

  // Stage a segment's activations (x rows in phase A, h rows in phase B) in the
  // block fixed-point layout.  Four consecutive threads share a chunk, one per
  // 8-column quarter.  Whole CTA; called between barriers.
  auto stage_x = [&](bool phase_b, int sg) {
    const int D = phase_b ? a.I : a.H;
    const int R = phase_b ? G.rounds_b : G.rounds_a;
    const int nch = D / 32, nt = seg_nt[sg], p0 = seg_pos[sg];
    const unsigned gmask = 0xfu << (lane & ~3);
    for (int task = threadIdx.x; task < nt * nch * 4; task += kThreads) {
      const int m = task & 3, tc = task >> 2, t = tc / nch, ch = tc % nch;
      const uint16_t* row = phase_b ? a.h + (size_t)(p0 + t) * a.I
                                    : a.x + (size_t)(plist[p0 + t] / a.k) * a.H;
      // L2 only: h comes from other CTAs
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(row + ch * 32 + m * 8));
      uint4 packed;
      const float2 sc = fixed_point_quarter(v, gmask, packed);
      const int i = ch / 32, l = ch % 32;
      xq[((size_t)(t * R + i) * 4 + m) * 32 + l] = packed;
      if (m == 0) xsc[t * R * 32 + ch] = sc;
    }
  };

  // out rows of the row blocks comb[0..n) for every token:
  // sum_j w[t,j] * y[pos(t,j)][c], j ascending.  One flat loop, so the loads of all
  // row blocks are in flight together.
  auto combine = [&](int n) {
    const int per_rb = a.T * G.rows_b;
    for (int e = threadIdx.x; e < n * per_rb; e += kThreads) {
      const int rb = comb[e / per_rb], rem = e % per_rb;
      const int t = rem / G.rows_b, c = rb * G.rows_b + rem % G.rows_b;
      if (c >= a.H) continue;
      float acc = 0.f;
      for (int j = 0; j < a.k; ++j) {
        const int p = t * a.k + j;
        const int pos = pos_of[p];
        if (pos >= 0) acc = fmaf(__ldg(a.w + p), __ldcg(a.y + (size_t)pos * a.H + c), acc);
      }
      a.out[(size_t)t * a.H + c] = float_to_bf16_bits(acc);
    }
  };

  // Publish the blocks of the segment just finished: phase A adds its block count to
  // hdone[seg]; phase B adds 1 to ydone[rb] for each of its row blocks, and the CTA
  // that completes the last segment of a row block combines it.  Whole CTA.
  int seg_open = -1, seg_phase = 0, seg_cnt = 0, rb_first = 0;
  auto publish = [&]() {
    if (seg_open < 0) return;
    __syncthreads();  // every warp's h / y stores of this segment are done
    if (seg_phase == 0) {
      // one thread releases the block's stores device-wide (the fence is cumulative
      // over what the barrier ordered before it) and counts them; nobody waits
      if (threadIdx.x == 0) {
        __threadfence();
        red_release_gpu(&hdone[seg_open], (unsigned)seg_cnt);
      }
      seg_open = -1;
      return;
    }
    if (warp == 0) {  // one lane per row block: the atomics overlap
      if (lane == 0) s_ncomb = 0;
      __syncwarp();
      __threadfence();
      for (int rb = rb_first + lane; rb < rb_first + seg_cnt; rb += 32) {
        const unsigned old = atomicAdd(&ydone[rb], 1u);
        if (old == (unsigned)nseg - 1) {
          ydone[rb] = 0;  // every segment of this row block is in: reset for the next call
          comb[atomicAdd(&s_ncomb, 1)] = rb;
        }
      }
      __threadfence();
    }
    __syncthreads();
    combine(s_ncomb);
    seg_open = -1;
  };

  int cur_seg_key = -1;
  for (int gi = 0; gi < ng; ++gi) {
    const bool phase_b = gi >= na;
    int sg, row0, nrows;
    if (!phase_b) {
      const int blk = a0 + gi;
      sg = blk / bpe_a;
      row0 = (blk % bpe_a) * kRowsA;
      nrows = kRowsA;
    } else {
      const int blk = b0 + (gi - na);
      sg = blk / bpe_b;
      row0 = (blk % bpe_b) * G.rows_b;
      nrows = min(G.rows_b, a.H - row0);
    }
    const int key = (phase_b ? 1 : 0) * kMaxPairsFused + sg;
    if (key != cur_seg_key) {  // new segment: publish the old one, swap the activations
      publish();
      if (phase_b && threadIdx.x == 0) wait_counter(&hdone[sg], (unsigned)bpe_a);
      __syncthreads();
      stage_x(phase_b, sg);
      __syncthreads();
      cur_seg_key = key;
      seg_open = sg;
      seg_phase = phase_b ? 1 : 0;
      seg_cnt = 0;
      rb_first = phase_b ? (b0 + (gi - na)) % bpe_b : 0;
    }
    ++seg_cnt;
    const int nt = seg_nt[sg], p0 = seg_pos[sg];
    const int st = gi % kStages;
    const bool ok = mbar_wait(&full[st], (gi / kStages) & 1);
    const unsigned char* buf = smem + L.stages + (size_t)st * G.stage_bytes;

    float Gs[kNT], Us[kNT];
    float v = 0.f;
    int vid = -1;
    if (ok && !phase_b) {
      const unsigned char* bgq = buf + (size_t)warp * (a.H / 2);
      const uint16_t* bgs = reinterpret_cast<const uint16_t*>(buf + G.a_q) + warp * (a.H / 64);
      const uint16_t* bgb = reinterpret_cast<const uint16_t*>(buf + G.a_q + G.a_sb) + warp * (a.H / 64);
      const unsigned char* bu = buf + G.a_mat;
      const unsigned char* buq = bu + (size_t)warp * (a.H / 2);
      const uint16_t* bus = reinterpret_cast<const uint16_t*>(bu + G.a_q) + warp * (a.H / 64);
      const uint16_t* bub = reinterpret_cast<const uint16_t*>(bu + G.a_q + G.a_sb) + warp * (a.H / 64);
      switch (nt) {
        case 1: dispatch_a<1>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, xq, xsc, lane, Gs, Us); break;
        case 2: dispatch_a<2>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, xq, xsc, lane, Gs, Us); break;
        case 3: dispatch_a<3>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, xq, xsc, lane, Gs, Us); break;
        default: dispatch_a<4>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, xq, xsc, lane, Gs, Us); break;
      }
    } else if (ok) {
      const uint16_t* bs = reinterpret_cast<const uint16_t*>(buf + G.b_q);
      const uint16_t* bb = reinterpret_cast<const uint16_t*>(buf + G.b_q + G.b_sb);
      switch (nt) {
        case 1: v = dispatch_b<1>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, xq, xsc, lane, vid); break;
        case 2: v = dispatch_b<2>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, xq, xsc, lane, vid); break;
        case 3: v = dispatch_b<3>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, xq, xsc, lane, vid); break;
        default: v = dispatch_b<4>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, xq, xsc, lane, vid); break;
      }
    }
    // this warp is done reading stage st; the last warp to get here refills it
    __threadfence_block();
    __syncwarp();
    if (lane == 0) {
      const int done = atomicAdd(&stage_cnt[st], 1);
      if (done == kWarps - 1) {
        stage_cnt[st] = 0;
        __threadfence_block();
        fence_proxy_async();
        if (gi + kStages < ng) issue(gi + kStages);
      }
    }
    if (ok && !phase_b) {
      if (lane < nt) {
        float gv = 0.f, uv = 0.f;
#pragma unroll
        for (int t = 0; t < kNT; ++t)
          if (t == lane) {
            gv = Gs[t];
            uv = Us[t];
          }
        const float g = round_to_bf16(gv), hu = round_to_bf16(uv);
        const float hv = g / (1.0f + __expf(-g)) * hu;
        a.h[(size_t)(p0 + lane) * a.I + row0 + warp] = float_to_bf16_bits(hv);
      }
    } else if (ok && vid >= 0) {
      const int r = warp + kWarps * (vid / kNT), t = vid % kNT;
      if (r < nrows) a.y[(size_t)(p0 + t) * a.H + row0 + r] = v;
    }
  }
  publish();
  if (nseg == 0) {  // nothing routed anywhere valid: every output row is zero
    const long long total = (long long)a.T * a.H;
    const long long o0 = total * blockIdx.x / gridDim.x, o1 = total * (blockIdx.x + 1) / gridDim.x;
    for (long long o = o0 + threadIdx.x; o < o1; o += kThreads) a.out[o] = 0;
  }
  grid_dep_launch();

  // ---- the CTA that finishes last resets the per-segment counters ----
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(exit_cnt, 1u);
    if (old == gridDim.x - 1) {
      for (int sgi = 0; sgi < nseg; ++sgi) hdone[sgi] = 0;
      *exit_cnt = 0;
      __threadfence();
    }
  }
}

}  // namespace qeg
