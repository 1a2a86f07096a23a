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
// The segment's activations sit in shared memory as fp32, laid out so that the
// 32 lanes of a warp read 512 consecutive bytes (no bank conflicts), with the
// per-chunk sums of x alongside.  A warp reduces its rows over its lanes once
// per block; there is no cross-warp exchange inside a phase.
//
// Codes become floats without integer->float conversion: nibble j of a word
// under exponent (150 - 4j) reads as 2^(23-4j) + q exactly; one packed fp32 add
// removes the offset.  Products q*x are exact in fp32; sums are fp32.
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
constexpr unsigned kXBytes = 64 * 1024;  // activation buffer (fp32)

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
  int s = (int)(kXBytes / (4096u * (unsigned)rmax));  // fp32 activations: rounds * 4 KB per pair
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
  s.cnt = align_up(s.xsum + sizeof(float) * kNT * rmax * 32, 16);
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

// ------------------------------------------------------------ code decode ---
// Masks, exponent fields and offsets of the decode.  Masks and exponents are kept
// in registers (hidden from constant folding) so that each nibble costs exactly
// one LOP3, (w & mask) | exponent.
struct DecodeConsts {
  uint32_t m0, m1, m2, m3, m4;            // 0xF << 4j, j = 0..4
  uint32_t e150, e146, e142, e138, e134;  // exponent (150 - 4j) << 23
  float2 c01, c23, c45, c67;
};
__device__ __forceinline__ DecodeConsts decode_consts() {
  DecodeConsts k;
  k.m0 = 0xFu;
  k.m1 = 0xF0u;
  k.m2 = 0xF00u;
  k.m3 = 0xF000u;
  k.m4 = 0xF0000u;
  k.e150 = 150u << 23;
  k.e146 = 146u << 23;
  k.e142 = 142u << 23;
  k.e138 = 138u << 23;
  k.e134 = 134u << 23;
  asm volatile("" : "+r"(k.m0), "+r"(k.m1), "+r"(k.m2), "+r"(k.m3), "+r"(k.m4));
  asm volatile("" : "+r"(k.e150), "+r"(k.e146), "+r"(k.e142), "+r"(k.e138), "+r"(k.e134));
  k.c01 = make_float2(-8388608.f, -524288.f);
  k.c23 = make_float2(-32768.f, -2048.f);
  k.c45 = make_float2(-128.f, -32768.f);
  k.c67 = make_float2(-2048.f, -128.f);
  return k;
}

// (a & b) | c in one instruction.
__device__ __forceinline__ float and_or_f(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return __uint_as_float(d);
}

// 8 codes of `w` (nibble j = element j) -> 4 float2 pairs (q0,q1) (q2,q3) (q4,q5) (q6,q7).
__device__ __forceinline__ void decode8(uint32_t w, const DecodeConsts& k, float2* q) {
  const uint32_t w2 = w >> 12;
  q[0] = __fadd2_rn(make_float2(and_or_f(w, k.m0, k.e150), and_or_f(w, k.m1, k.e146)), k.c01);
  q[1] = __fadd2_rn(make_float2(and_or_f(w, k.m2, k.e142), and_or_f(w, k.m3, k.e138)), k.c23);
  q[2] = __fadd2_rn(make_float2(and_or_f(w, k.m4, k.e134), and_or_f(w2, k.m2, k.e142)), k.c45);
  q[3] = __fadd2_rn(make_float2(and_or_f(w2, k.m3, k.e138), and_or_f(w2, k.m4, k.e134)), k.c67);
}

// The 32 codes of a uint4 (elements 8i + j = nibble j of word i) as 16 float2 pairs.
__device__ __forceinline__ void decode32(const uint4 v, const DecodeConsts& k, float2 (&q)[16]) {
  decode8(v.x, k, &q[0]);
  decode8(v.y, k, &q[4]);
  decode8(v.z, k, &q[8]);
  decode8(v.w, k, &q[12]);
}

// sum_c q_c x_c over one 32-column chunk: x as 8 float4 (columns 4j..4j+3).
__device__ __forceinline__ float dot32(const float2 (&q)[16], const float4 (&x)[8]) {
  float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    a = __ffma2_rn(q[2 * j], make_float2(x[j].x, x[j].y), a);
    b = __ffma2_rn(q[2 * j + 1], make_float2(x[j].z, x[j].w), b);
  }
  return (a.x + a.y) + (b.x + b.y);
}

// Activation buffer layout: float4 (t, round i, j, lane) at ((t*R + i)*8 + j)*32 + lane
// holds columns (i*32 + lane)*32 + 4j .. +3; chunk sums at t*R*32 + i*32 + lane.
__device__ __forceinline__ void load_xchunk(const float4* xs4, int t, int R, int i, int lane,
                                            float4 (&x)[8]) {
  const float4* p = xs4 + ((size_t)(t * R + i) * 8) * 32 + lane;
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = p[j * 32];
}

// ---------------------------------------------------------------- counters ---
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
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
// (chunks past H/32 skipped); returns (G, U) for t < NT in every lane.
template <int NT, int R>
__device__ __forceinline__ void rows_a(const unsigned char* bg_q, const uint16_t* bg_s,
                                       const uint16_t* bg_b, const unsigned char* bu_q,
                                       const uint16_t* bu_s, const uint16_t* bu_b, int H,
                                       const float4* xs4, const float* xsum, int lane,
                                       const DecodeConsts& k, float (&G)[kNT],
                                       float (&U)[kNT]) {
  float ag[NT], au[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) ag[t] = au[t] = 0.f;
  const int nch = H / 32;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int ch = i * 32 + lane;
    if (ch < nch) {
      const uint4 vg = *reinterpret_cast<const uint4*>(bg_q + ch * 16);
      const uint4 vu = *reinterpret_cast<const uint4*>(bu_q + ch * 16);
      const float sg = bf16_bits_to_float(bg_s[ch >> 1]), bgv = bf16_bits_to_float(bg_b[ch >> 1]);
      const float su = bf16_bits_to_float(bu_s[ch >> 1]), buv = bf16_bits_to_float(bu_b[ch >> 1]);
      float2 qg[16], qu[16];
      decode32(vg, k, qg);
      decode32(vu, k, qu);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float4 x[8];
        load_xchunk(xs4, t, R, i, lane, x);
        const float xsv = xsum[t * R * 32 + ch];
        ag[t] += fmaf(sg, dot32(qg, x), bgv * xsv);
        au[t] += fmaf(su, dot32(qu, x), buv * xsv);
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
// Per 32-column round the activations of all NT pairs are loaded once, then each
// row is decoded once and dotted with them.  Returns the value this lane holds
// after a reduce-scatter and its index q*kNT + t in `vid` (-1 when it holds none).
template <int NT, int R>
__device__ __forceinline__ float rows_b(const unsigned char* bq, const uint16_t* bs,
                                        const uint16_t* bb, int row0, int nrows, int I,
                                        const float4* xs4, const float* xsum, int lane,
                                        const DecodeConsts& k, int& vid) {
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
      float4 x[NT][8];
      float xsv[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        load_xchunk(xs4, t, R, i, lane, x[t]);
        xsv[t] = xsum[t * R * 32 + ch];
      }
#pragma unroll
      for (int q = 0; q < kMaxRowsPerWarpB; ++q) {
        const int r = row0 + kWarps * q;
        if (r < nrows) {
          const uint4 v = *reinterpret_cast<const uint4*>(bq + (size_t)r * qstride + ch * 16);
          const float sc = bf16_bits_to_float(bs[r * sstride + (ch >> 1)]);
          const float bi = bf16_bits_to_float(bb[r * sstride + (ch >> 1)]);
          float2 qd[16];
          decode32(v, k, qd);
#pragma unroll
          for (int t = 0; t < NT; ++t) acc[q * NP + t] += fmaf(sc, dot32(qd, x[t]), bi * xsv[t]);
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
                                           const float4* xs4, const float* xsum, int lane,
                                           const DecodeConsts& k, float (&G)[kNT],
                                           float (&U)[kNT]) {
  if (R == 1) rows_a<NT, 1>(bgq, bgs, bgb, buq, bus, bub, H, xs4, xsum, lane, k, G, U);
  else if (R == 2) rows_a<NT, 2>(bgq, bgs, bgb, buq, bus, bub, H, xs4, xsum, lane, k, G, U);
  else rows_a<NT, 4>(bgq, bgs, bgb, buq, bus, bub, H, xs4, xsum, lane, k, G, U);
}

template <int NT>
__device__ __forceinline__ float dispatch_b(int R, const unsigned char* bq, const uint16_t* bs,
                                            const uint16_t* bb, int row0, int nrows, int I,
                                            const float4* xs4, const float* xsum, int lane,
                                            const DecodeConsts& k, int& vid) {
  if (R == 1) return rows_b<NT, 1>(bq, bs, bb, row0, nrows, I, xs4, xsum, lane, k, vid);
  if (R == 2) return rows_b<NT, 2>(bq, bs, bb, row0, nrows, I, xs4, xsum, lane, k, vid);
  if (R == 4) return rows_b<NT, 4>(bq, bs, bb, row0, nrows, I, xs4, xsum, lane, k, vid);
  return rows_b<NT, 8>(bq, bs, bb, row0, nrows, I, xs4, xsum, lane, k, vid);
}

__global__ void __launch_bounds__(kThreads, 1) layer_kernel(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_u, s_nseg, s_ncomb;
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
  const int bpe_a = a.I / kRowsA;
  const int bpe_b = (a.H + G.rows_b - 1) / G.rows_b;
  const long long na_tot = (long long)nseg * bpe_a, nb_tot = (long long)nseg * bpe_b;
  const int a0 = (int)(na_tot * blockIdx.x / gridDim.x);
  const int na = (int)(na_tot * (blockIdx.x + 1) / gridDim.x) - a0;
  const int b0 = (int)(nb_tot * blockIdx.x / gridDim.x);
  const int nb = (int)(nb_tot * (blockIdx.x + 1) / gridDim.x) - b0;
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
  if (threadIdx.x == 0)
    for (int gi = 0; gi < ng && gi < kStages; ++gi) issue(gi);

  if (blockIdx.x == 0 && warp == 1 && a.ex_u) {
    for (int i = lane; i < u; i += 32) a.ex_unique[i] = uniq[i];
    for (int i = lane; i <= u; i += 32) a.ex_offsets[i] = offs[i];
    for (int i = lane; i < P; i += 32) a.ex_pair_list[i] = plist[i];
    if (lane == 0) *a.ex_u = u;
  }

  float4* xs4 = reinterpret_cast<float4*>(smem + L.x);
  float* xsum = reinterpret_cast<float*>(smem + L.xsum);
  const DecodeConsts dk = decode_consts();

  // Stage a segment's activations (x rows in phase A, h rows in phase B) as fp32 in
  // the shared buffer, with per-chunk sums.  Whole CTA; called between barriers.
  auto stage_x = [&](bool phase_b, int sg) {
    const int D = phase_b ? a.I : a.H;
    const int R = phase_b ? G.rounds_b : G.rounds_a;
    const int nch = D / 32, nt = seg_nt[sg], p0 = seg_pos[sg];
    for (int task = threadIdx.x; task < nt * nch; task += kThreads) {
      const int t = task / nch, ch = task % nch;
      const uint16_t* row = phase_b ? a.h + (size_t)(p0 + t) * a.I
                                    : a.x + (size_t)(plist[p0 + t] / a.k) * a.H;
      const uint4* src = reinterpret_cast<const uint4*>(row + ch * 32);
      uint4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = __ldcg(src + q);  // L2: h comes from other CTAs
      const int i = ch / 32, l = ch % 32;
      float4* dst = xs4 + ((size_t)(t * R + i) * 8) * 32 + l;
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t w4[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
        const float4 f0 = make_float4(bf16_lo(w4[0]), bf16_hi(w4[0]), bf16_lo(w4[1]), bf16_hi(w4[1]));
        const float4 f1 = make_float4(bf16_lo(w4[2]), bf16_hi(w4[2]), bf16_lo(w4[3]), bf16_hi(w4[3]));
        dst[(2 * q) * 32] = f0;
        dst[(2 * q + 1) * 32] = f1;
        sum += (f0.x + f0.y) + (f0.z + f0.w) + (f1.x + f1.y) + (f1.z + f1.w);
      }
      xsum[t * R * 32 + ch] = sum;
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
    __threadfence();  // this thread's h / y stores are visible device-wide
    __syncthreads();
    if (threadIdx.x == 0) {
      s_ncomb = 0;
      if (seg_phase == 0) atomicAdd(&hdone[seg_open], (unsigned)seg_cnt);
    }
    __syncthreads();
    if (seg_phase == 1 && warp == 0) {  // one lane per row block: the atomics overlap
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
        case 1: dispatch_a<1>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, xs4, xsum, lane, dk, Gs, Us); break;
        case 2: dispatch_a<2>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, xs4, xsum, lane, dk, Gs, Us); break;
        case 3: dispatch_a<3>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, xs4, xsum, lane, dk, Gs, Us); break;
        default: dispatch_a<4>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, xs4, xsum, lane, dk, Gs, Us); break;
      }
    } else if (ok) {
      const uint16_t* bs = reinterpret_cast<const uint16_t*>(buf + G.b_q);
      const uint16_t* bb = reinterpret_cast<const uint16_t*>(buf + G.b_q + G.b_sb);
      switch (nt) {
        case 1: v = dispatch_b<1>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, xs4, xsum, lane, dk, vid); break;
        case 2: v = dispatch_b<2>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, xs4, xsum, lane, dk, vid); break;
        case 3: v = dispatch_b<3>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, xs4, xsum, lane, dk, vid); break;
        default: v = dispatch_b<4>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, xs4, xsum, lane, dk, vid); break;
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
