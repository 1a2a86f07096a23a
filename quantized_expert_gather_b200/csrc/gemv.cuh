// Expert-major dequant-GEMV kernels for small token windows (T <= 256).
//
// K2 (gate_up_kernel): for every distinct routed expert e, stream Wg[e] and
//   Wu[e] from HBM once, in blocks of kRows rows, through a kStages-deep ring of
//   shared-memory buffers filled by 1-D bulk copies (mbarrier completion).
//   Thread 0 issues the copies: the first kStages blocks up front, then block
//   j + kStages right after the barrier that ends block j, when no warp reads
//   its slot any more.  Every warp computes; blocks have 8 warps at most, so
//   each SM sub-partition holds two and a thread may use up to 255 registers.
//   The warps hold the activations of the expert's
//   tokens in registers and compute, per row and token,
//     G = sum_c (s*q_c + b) x_c = s * sum_c q_c x_c + b * sum_c x_c
//   (group-sum factorisation over the 32 columns a lane owns, one group), then
//   h = bf16(silu(bf16 G) * bf16 U), the one-pass epilogue of "Apple7/8 MoE gate
//   and up in one decode pass" (splash PR 45, "What changed").  h is written
//   in pair_list order.
// K3 (down_combine_kernel): each CTA owns a block of output rows; it streams
//   those rows of Wd[e] for every distinct expert in ascending order, computes
//   y = Wd[e] h for the expert's pairs and adds w * y into per-token fp32
//   accumulators in that fixed order, then writes bf16 out.  No atomics: the
//   combine order is the same on every run.
//
// Codes are turned into floats without integer->float conversions: nibble j of
// a word placed under exponent (150 - 4j) reads as 2^(23-4j) + q exactly, and
// one packed fp32 add removes the offset.  Products q*x are exact in fp32.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "union.cuh"

namespace qeg {

constexpr int kRows = 8;       // K2: rows of gate and of up per stage
constexpr int kStages2 = 4;    // K2: ring depth
constexpr int kStages3 = 5;    // K3: ring depth
constexpr int kNT = 4;         // tokens (pairs) per register pass
constexpr int kConsWarps = 8;  // warps per CTA (K2 at hidden 4096, K3); all compute
constexpr int kThreads = 32 * kConsWarps;
constexpr int kRowsPerWarp3 = 8;  // K3: output rows per consumer warp
constexpr int kMaxRows3 = kConsWarps * kRowsPerWarp3;  // K3: output rows per CTA at most
constexpr int kGemvMaxT = 256;
constexpr int kGemvMaxPairs = 2048;

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------ smem layouts ---
struct UnionSmem {
  size_t cnt, rank, unique, offsets, pair_list, end;
};
__host__ __device__ inline UnionSmem union_smem(size_t base, int E, int P) {
  UnionSmem u;
  const int m = (E < P ? E : P) > 0 ? (E < P ? E : P) : 1;
  u.cnt = base;
  u.rank = align_up(u.cnt + sizeof(int) * E, 16);
  u.unique = align_up(u.rank + sizeof(int) * P, 16);
  u.offsets = align_up(u.unique + sizeof(int) * m, 16);
  u.pair_list = align_up(u.offsets + sizeof(int) * (m + 1), 16);
  u.end = align_up(u.pair_list + sizeof(int) * (P > 0 ? P : 1), 16);
  return u;
}

struct K2Layout {
  unsigned q_bytes, sb_bytes, mat_bytes, stage_bytes;
  size_t bars, stages, part, uni, total;
  UnionSmem us;
};
__host__ __device__ inline K2Layout k2_layout(int H, int E, int P, int ncw) {
  K2Layout L;
  L.q_bytes = kRows * H / 2;
  L.sb_bytes = kRows * H / 32;
  L.mat_bytes = L.q_bytes + 2 * L.sb_bytes;
  L.stage_bytes = 2 * L.mat_bytes;
  L.bars = 0;  // (barriers live in static shared memory)
  L.stages = 128;
  L.part = L.stages + align_up((size_t)kStages2 * L.stage_bytes, 128);
  // partials: [2 buffers][2 matrices][ncw][kRows * kNT] floats
  L.uni = align_up(L.part + sizeof(float) * 2 * 2 * ncw * kRows * kNT, 128);
  L.us = union_smem(L.uni, E, P);
  L.total = L.us.end;
  return L;
}

struct K3Layout {
  unsigned q_bytes, sb_bytes, stage_bytes;
  size_t stages, part, acc, uni, total;
  UnionSmem us;
};
__host__ __device__ inline K3Layout k3_layout(int I, int E, int P, int T, int ncw3,
                                              int rows_per_cta) {
  K3Layout L;
  L.q_bytes = rows_per_cta * I / 2;
  L.sb_bytes = rows_per_cta * I / 32;
  L.stage_bytes = L.q_bytes + 2 * L.sb_bytes;
  L.stages = 128;
  L.part = L.stages + align_up((size_t)kStages3 * L.stage_bytes, 128);
  // partials: [2][ncw3][kMaxRows3][kNT]; acc: [T][rows_per_cta].  ncw3 chunk-warps
  // split a row; kConsWarps / ncw3 row groups split the CTA's rows.
  L.acc = align_up(L.part + sizeof(float) * 2 * ncw3 * kMaxRows3 * kNT, 128);
  L.uni = align_up(L.acc + sizeof(float) * (size_t)T * rows_per_cta, 128);
  L.us = union_smem(L.uni, E, P);
  L.total = L.us.end;
  return L;
}

// -------------------------------------------------------------- arguments ---
struct UnionGlobal {      // route-union produced by the route_union kernel
  const int* num_unique;  // null: compute the union in shared memory
  const int* unique;
  const int* offsets;
  const int* pair_list;
};

struct GateUpArgs {
  const uint16_t* x;
  const int* idx;
  const uint32_t *gq, *uq;
  const uint16_t *gs, *gb, *us, *ub;
  uint16_t* h;  // [P, I] bf16, rows in pair_list order
  UnionGlobal ug;
  int *ex_u, *ex_unique, *ex_offsets, *ex_pair_list;  // optional export of the union (CTA 0)
  int T, k, E, H, I, ncw;
  int wait_prior;  // wait for the preceding grid before reading any input
};

struct DownArgs {
  const int* idx;
  const float* w;
  const uint32_t* dq;
  const uint16_t *ds, *db;
  const uint16_t* h;
  uint16_t* out;
  UnionGlobal ug;
  int T, k, E, H, I, ncw3, rows_per_cta;
};

// ------------------------------------------------------------ code decode ---
// 8 codes of `w` (nibble j = element j) -> 4 float2 pairs (q0,q1) (q2,q3) (q4,q5) (q6,q7).
__device__ __forceinline__ void decode8(uint32_t w, float2 (&q)[4]) {
  const uint32_t w2 = w >> 12;
  const float a0 = __uint_as_float((150u << 23) | (w & 0xFu));
  const float a1 = __uint_as_float((146u << 23) | (w & 0xF0u));
  const float a2 = __uint_as_float((142u << 23) | (w & 0xF00u));
  const float a3 = __uint_as_float((138u << 23) | (w & 0xF000u));
  const float a4 = __uint_as_float((134u << 23) | (w & 0xF0000u));
  const float a5 = __uint_as_float((142u << 23) | (w2 & 0xF00u));
  const float a6 = __uint_as_float((138u << 23) | (w2 & 0xF000u));
  const float a7 = __uint_as_float((134u << 23) | (w2 & 0xF0000u));
  q[0] = __fadd2_rn(make_float2(a0, a1), make_float2(-8388608.f, -524288.f));
  q[1] = __fadd2_rn(make_float2(a2, a3), make_float2(-32768.f, -2048.f));
  q[2] = __fadd2_rn(make_float2(a4, a5), make_float2(-128.f, -32768.f));
  q[3] = __fadd2_rn(make_float2(a6, a7), make_float2(-2048.f, -128.f));
}

// Load the 32 activations a lane owns (chunk `ch` of a row) as fp32 and their sum.
__device__ __forceinline__ void load_x32(const uint16_t* __restrict__ row, int ch, float (&xf)[32],
                                         float& xs) {
  const uint4* p = reinterpret_cast<const uint4*>(row + ch * 32);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = __ldcg(p + i);  // L2 only: data may come from the preceding grid
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      xf[i * 8 + 2 * j] = bf16_lo(u[j]);
      xf[i * 8 + 2 * j + 1] = bf16_hi(u[j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) s += xf[i];
  xs = s;
}

// acc[t] = sum over the 32 codes of `wv` of q_c * x_t[c], for t < nt.
__device__ __forceinline__ void dot32(const uint4 wv, const float (&xf)[kNT][32], int nt,
                                      float (&dot)[kNT]) {
  float2 a[kNT];
#pragma unroll
  for (int t = 0; t < kNT; ++t) a[t] = make_float2(0.f, 0.f);
  const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 q[4];
    decode8(ws[i], q);
#pragma unroll
    for (int t = 0; t < kNT; ++t) {
      if (t < nt) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          a[t] = __ffma2_rn(q[j], make_float2(xf[t][i * 8 + 2 * j], xf[t][i * 8 + 2 * j + 1]),
                            a[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kNT; ++t) dot[t] = a[t].x + a[t].y;
}

// Resolve the union either from global arrays (route_union kernel output) or by
// computing it in shared memory with warp 0.  All threads call this.
struct UnionRefs {
  int u;
  const int* unique;
  const int* offsets;
  const int* pair_list;
};

__device__ __forceinline__ UnionRefs block_union(const UnionGlobal& ug, const int* idx, int P,
                                                 int E, unsigned char* smem, const UnionSmem& us,
                                                 int* s_u) {
  UnionRefs r;
  if (ug.num_unique) {
    r.u = *ug.num_unique;
    r.unique = ug.unique;
    r.offsets = ug.offsets;
    r.pair_list = ug.pair_list;
    return r;
  }
  int* cnt = reinterpret_cast<int*>(smem + us.cnt);
  int* rank = reinterpret_cast<int*>(smem + us.rank);
  int* uniq = reinterpret_cast<int*>(smem + us.unique);
  int* offs = reinterpret_cast<int*>(smem + us.offsets);
  int* plist = reinterpret_cast<int*>(smem + us.pair_list);
  if (threadIdx.x < 32) {
    int nv;
    const int u = warp_route_union(idx, P, E, cnt, rank, uniq, offs, plist, &nv);
    if (threadIdx.x == 0) *s_u = u;
  }
  __syncthreads();
  r.u = *s_u;
  r.unique = uniq;
  r.offsets = offs;
  r.pair_list = plist;
  return r;
}

// Copy a shared-memory union to global memory (for inspection); one warp.
__device__ __forceinline__ void export_union(const UnionRefs& U, int P, int* g_u, int* g_unique,
                                             int* g_offsets, int* g_pair_list) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < U.u; i += 32) g_unique[i] = U.unique[i];
  for (int i = lane; i <= U.u; i += 32) g_offsets[i] = U.offsets[i];
  for (int i = lane; i < P; i += 32) g_pair_list[i] = U.pair_list[i];
  if (lane == 0) *g_u = U.u;
}

// ------------------------------------------------------------------- K2 ---
__global__ void __launch_bounds__(kThreads, 1) gate_up_kernel(const GateUpArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_u;
  __shared__ __align__(8) uint64_t full[kStages2];
  const int P = a.T * a.k;
  const K2Layout L = k2_layout(a.H, a.E, P, a.ncw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_threads = 2 * a.ncw * 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
  }
  if (a.wait_prior) grid_dep_wait();
  const UnionRefs U = block_union(a.ug, a.idx, P, a.E, smem, L.us, &s_u);
  __syncthreads();  // barrier init and union visible to every warp
  grid_dep_launch();
  if (blockIdx.x == 0 && warp == 1 && a.ex_u && !a.ug.num_unique)
    export_union(U, P, a.ex_u, a.ex_unique, a.ex_offsets, a.ex_pair_list);

  const int bpe = a.I / kRows;  // row blocks per expert
  const long long nb = (long long)U.u * bpe;
  const int blk0 = (int)(nb * blockIdx.x / gridDim.x);
  const int blk1 = (int)(nb * (blockIdx.x + 1) / gridDim.x);
  const int nblk = blk1 - blk0;
  const size_t qrow = a.H / 8, srow = a.H / 64;  // words / groups per row
  uint64_t pol = 0;

  // thread 0: copy row block j of this CTA's range into ring slot j % kStages2
  auto issue = [&](int j) {
    const int blk = blk0 + j, slot = blk / bpe, row0 = (blk % bpe) * kRows;
    const int st = j % kStages2;
    unsigned char* buf = smem + L.stages + (size_t)st * L.stage_bytes;
    const size_t r0 = (size_t)U.unique[slot] * a.I + row0;
    mbar_arrive_expect_tx(&full[st], L.stage_bytes);
    bulk_g2s(buf, a.gq + r0 * qrow, L.q_bytes, &full[st], pol);
    bulk_g2s(buf + L.q_bytes, a.gs + r0 * srow, L.sb_bytes, &full[st], pol);
    bulk_g2s(buf + L.q_bytes + L.sb_bytes, a.gb + r0 * srow, L.sb_bytes, &full[st], pol);
    buf += L.mat_bytes;
    bulk_g2s(buf, a.uq + r0 * qrow, L.q_bytes, &full[st], pol);
    bulk_g2s(buf + L.q_bytes, a.us + r0 * srow, L.sb_bytes, &full[st], pol);
    bulk_g2s(buf + L.q_bytes + L.sb_bytes, a.ub + r0 * srow, L.sb_bytes, &full[st], pol);
  };
  if (threadIdx.x == 0) {
    pol = policy_evict_first();
    for (int j = 0; j < nblk && j < kStages2; ++j) issue(j);
  }

  const int m = warp / a.ncw, cw = warp % a.ncw;  // matrix (0 gate, 1 up), chunk-warp
  const int ch = cw * 32 + lane;
  const bool active = ch < a.H / 32;
  float* part = reinterpret_cast<float*>(smem + L.part);
  const int part_stride = 2 * a.ncw * kRows * kNT;  // one buffer
  const int ct = threadIdx.x;
  float xf[kNT][32];
  float xs[kNT];
  int cur_slot = -1, cur_c0 = -1;
  int pb = 0;

  for (int j = 0; j < nblk; ++j) {
    const int blk = blk0 + j, slot = blk / bpe, row0 = (blk % bpe) * kRows;
    const int st = j % kStages2;
    const int pos0 = U.offsets[slot], n_e = U.offsets[slot + 1] - pos0;
    const bool ok = mbar_wait(&full[st], (j / kStages2) & 1);
    const unsigned char* buf = smem + L.stages + (size_t)st * L.stage_bytes + m * L.mat_bytes;
    const unsigned char* bq = buf;
    const uint16_t* bs = reinterpret_cast<const uint16_t*>(buf + L.q_bytes);
    const uint16_t* bb = reinterpret_cast<const uint16_t*>(buf + L.q_bytes + L.sb_bytes);
    for (int c0 = 0; c0 < n_e; c0 += kNT) {
      const int nt = min(kNT, n_e - c0);
      if (slot != cur_slot || c0 != cur_c0) {
#pragma unroll
        for (int t = 0; t < kNT; ++t) {
          if (t < nt && active) {
            const int tok = U.pair_list[pos0 + c0 + t] / a.k;
            load_x32(a.x + (size_t)tok * a.H, ch, xf[t], xs[t]);
          }
        }
        cur_slot = slot;
        cur_c0 = c0;
      }
      float acc[kRows * kNT];
#pragma unroll
      for (int i = 0; i < kRows * kNT; ++i) acc[i] = 0.f;
      if (active && ok) {
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          const uint4 wv = *reinterpret_cast<const uint4*>(bq + (size_t)r * (a.H / 2) + ch * 16);
          const float sc = bf16_bits_to_float(bs[r * (a.H / 64) + (ch >> 1)]);
          const float bi = bf16_bits_to_float(bb[r * (a.H / 64) + (ch >> 1)]);
          float d[kNT];
          dot32(wv, xf, nt, d);
#pragma unroll
          for (int t = 0; t < kNT; ++t) acc[r * kNT + t] = fmaf(sc, d[t], bi * xs[t]);
        }
      }
      int vid;
      const float v = warp_reduce_scatter<kRows * kNT>(acc, lane, vid);
      float* pbuf = part + pb * part_stride;
      pbuf[(m * a.ncw + cw) * (kRows * kNT) + vid] = v;  // V == 32: every lane owns one value
      named_barrier(1, n_threads);
      // every warp is past its reads of slot st: refill it with block j + kStages2
      if (c0 + kNT >= n_e && threadIdx.x == 0 && j + kStages2 < nblk) {
        fence_proxy_async();
        issue(j + kStages2);
      }
      if (ct < kRows * nt) {
        const int r = ct / nt, t = ct % nt;
        float G = 0.f, Uv = 0.f;
        for (int c = 0; c < a.ncw; ++c) {
          G += pbuf[(0 * a.ncw + c) * (kRows * kNT) + r * kNT + t];
          Uv += pbuf[(1 * a.ncw + c) * (kRows * kNT) + r * kNT + t];
        }
        const float g = round_to_bf16(G), u = round_to_bf16(Uv);
        const float hv = g / (1.0f + __expf(-g)) * u;
        a.h[(size_t)(pos0 + c0 + t) * a.I + row0 + r] = float_to_bf16_bits(hv);
      }
      pb ^= 1;
    }
  }
}

// ------------------------------------------------------------------- K3 ---
__global__ void __launch_bounds__(kThreads, 1) down_combine_kernel(const DownArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_u;
  __shared__ __align__(8) uint64_t full[kStages3];
  const int P = a.T * a.k;
  const K3Layout L = k3_layout(a.I, a.E, P, a.T, a.ncw3, a.rows_per_cta);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_groups = kConsWarps / a.ncw3;
  const int c0row = blockIdx.x * a.rows_per_cta;
  const int nrows = min(a.rows_per_cta, a.H - c0row);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages3; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
  }
  float* acc_out = reinterpret_cast<float*>(smem + L.acc);
  for (int i = threadIdx.x; i < a.T * a.rows_per_cta; i += blockDim.x) acc_out[i] = 0.f;
  // The union depends only on topk_idx, which is ready before the preceding
  // grid (gate+up) started, so it is formed before waiting on that grid.
  const UnionRefs U = block_union(a.ug, a.idx, P, a.E, smem, L.us, &s_u);
  __syncthreads();  // barrier init, zeroed accumulators and union visible to every warp
  grid_dep_launch();
  const size_t qrow = a.I / 8, srow = a.I / 64;
  const unsigned q_bytes = nrows * (a.I / 2), sb_bytes = nrows * (a.I / 32);
  uint64_t pol = 0;

  // thread 0: copy this CTA's rows of Wd[unique[j]] into ring slot j % kStages3
  auto issue = [&](int j) {
    const int st = j % kStages3;
    unsigned char* buf = smem + L.stages + (size_t)st * L.stage_bytes;
    const size_t r0 = (size_t)U.unique[j] * a.H + c0row;
    mbar_arrive_expect_tx(&full[st], q_bytes + 2 * sb_bytes);
    bulk_g2s(buf, a.dq + r0 * qrow, q_bytes, &full[st], pol);
    bulk_g2s(buf + L.q_bytes, a.ds + r0 * srow, sb_bytes, &full[st], pol);
    bulk_g2s(buf + L.q_bytes + L.sb_bytes, a.db + r0 * srow, sb_bytes, &full[st], pol);
  };
  // Weights do not depend on the preceding grid: start streaming them now.
  if (threadIdx.x == 0) {
    pol = policy_evict_first();
    for (int j = 0; j < U.u && j < kStages3; ++j) issue(j);
  }
  // h comes from the preceding grid.
  grid_dep_wait();

  const int cw = warp % a.ncw3, rg = warp / a.ncw3;
  const int ch = cw * 32 + lane;
  const bool active = ch < a.I / 32;
  float* part = reinterpret_cast<float*>(smem + L.part);
  const int part_stride = a.ncw3 * kMaxRows3 * kNT;
  const int ct = threadIdx.x;
  float xf[kNT][32];
  float xs[kNT];
  int pb = 0;
  for (int j = 0; j < U.u; ++j) {
    const int st = j % kStages3;
    const int pos0 = U.offsets[j], n_e = U.offsets[j + 1] - pos0;
    const bool ok = mbar_wait(&full[st], (j / kStages3) & 1);
    const unsigned char* bq = smem + L.stages + (size_t)st * L.stage_bytes;
    const uint16_t* bs = reinterpret_cast<const uint16_t*>(bq + L.q_bytes);
    const uint16_t* bb = reinterpret_cast<const uint16_t*>(bq + L.q_bytes + L.sb_bytes);
    for (int c0 = 0; c0 < n_e; c0 += kNT) {
      const int nt = min(kNT, n_e - c0);
#pragma unroll
      for (int t = 0; t < kNT; ++t)
        if (t < nt && active) load_x32(a.h + (size_t)(pos0 + c0 + t) * a.I, ch, xf[t], xs[t]);
      float acc[kRowsPerWarp3 * kNT];
#pragma unroll
      for (int i = 0; i < kRowsPerWarp3 * kNT; ++i) acc[i] = 0.f;
      if (active && ok) {
#pragma unroll
        for (int i = 0; i < kRowsPerWarp3; ++i) {
          const int r = rg + row_groups * i;
          if (r < nrows) {
            const uint4 wv = *reinterpret_cast<const uint4*>(bq + (size_t)r * (a.I / 2) + ch * 16);
            const float sc = bf16_bits_to_float(bs[r * (a.I / 64) + (ch >> 1)]);
            const float bi = bf16_bits_to_float(bb[r * (a.I / 64) + (ch >> 1)]);
            float d[kNT];
            dot32(wv, xf, nt, d);
#pragma unroll
            for (int t = 0; t < kNT; ++t) acc[i * kNT + t] = fmaf(sc, d[t], bi * xs[t]);
          }
        }
      }
      int vid;
      const float v = warp_reduce_scatter<kRowsPerWarp3 * kNT>(acc, lane, vid);
      float* pbuf = part + pb * part_stride;
      {
        const int i = vid / kNT, t = vid % kNT;
        const int r = rg + row_groups * i;
        if (r < kMaxRows3) pbuf[(cw * kMaxRows3 + r) * kNT + t] = v;
      }
      named_barrier(1, kThreads);
      if (c0 + kNT >= n_e && threadIdx.x == 0 && j + kStages3 < U.u) {
        fence_proxy_async();
        issue(j + kStages3);
      }
      if (ct < nrows) {
        const int r = ct;
        for (int t = 0; t < nt; ++t) {
          float y = 0.f;
          for (int c = 0; c < a.ncw3; ++c) y += pbuf[(c * kMaxRows3 + r) * kNT + t];
          const int p = U.pair_list[pos0 + c0 + t];
          acc_out[(p / a.k) * a.rows_per_cta + r] += a.w[p] * y;
        }
      }
      pb ^= 1;
    }
  }
  named_barrier(1, kThreads);
  for (int i = ct; i < a.T * nrows; i += kThreads) {
    const int t = i / nrows, r = i % nrows;
    a.out[(size_t)t * a.H + c0row + r] = float_to_bf16_bits(acc_out[t * a.rows_per_cta + r]);
  }
}

}  // namespace qeg
