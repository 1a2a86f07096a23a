// Large-window path: the same layer as layer.cuh as grouped GEMMs on the 5th-
// generation tensor cores, for windows with more pairs than the persistent
// kernel holds.
//
// "MoE GatherQMM small-M verify cost" (llms-explorer fact sheet): above a pair
// threshold the pairs are sorted by expert and each expert's rows are applied as
// one matrix product (the sorted grouped path).  Here, after the route-union
// (route_union.cuh) has grouped the pairs by expert:
//
//   grouped_kernel<0>  gate+up: for each (expert slot, 128 rows of Wg/Wu) tile,
//                      G = Wg X^T and U = Wu X^T over the expert's tokens, with
//                      h = bf16(silu(bf16 G) * bf16 U) stored per pair;
//   grouped_kernel<1>  down: for each (expert slot, 128 rows of Wd) tile,
//                      Y = Wd H^T over the expert's pairs, fp32 per pair;
//   combine_kernel     out[t] = bf16(sum_j w[t,j] * y[t,j]), j ascending.
//
// A tile is M = 128 weight rows by N = the expert's pairs (at most 256 at a
// time, padded to a multiple of 16), K in slabs of 64.  Per slab all threads
// dequantise the 4-bit codes, w = s * q + b in fp32, and split each weight into
// two bf16 parts, hi = bf16(w) and lo = bf16(w - hi) (hi + lo holds w to about 16
// significant bits), and gather the activation rows (bf16, exact), all into
// 128-byte-swizzled K-major shared-memory tiles; one thread issues tcgen05.mma
// (bf16 x bf16, fp32 accumulator in tensor memory) for hi and for lo into the
// same accumulator and commits to an mbarrier.  Two slab buffers let
// the dequantisation of slab s+1 overlap the MMAs of slab s.  The epilogue warps
// read the accumulators with tcgen05.ld.
#pragma once

#include "common.cuh"

namespace qeg {

constexpr int kGThreads = 256;       // 8 warps
constexpr int kGM = 128;             // weight rows per tile (MMA M)
constexpr int kGMaxN = 256;          // pairs per MMA (MMA N, multiple of 16)
constexpr int kGK = 64;              // K per slab (one 128-byte swizzle row of bf16)
constexpr unsigned kGATile = kGM * kGK * 2;     // 16 KB: one matrix slab
constexpr unsigned kGBTile = kGMaxN * kGK * 2;  // 32 KB: activation slab
// dynamic shared memory: per buffer [A0hi | A0lo | A1hi | A1lo | B] (A1 only for
// gate+up), 2 buffers
constexpr unsigned kGSmem = 2 * (4 * kGATile + kGBTile) + 1024;  // + alignment slack

// ------------------------------------------------------------ tcgen05 helpers ---
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (both operands bf16).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The mbarrier receives one arrival when every MMA this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// 16 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled tile: rows of 128
// bytes (64 bf16 of K), 8-row groups 1024 bytes apart (stride byte offset), the
// tile based at a 1024-byte boundary; `addr` may be advanced by 32-byte K steps
// inside the row.  Fields: start address >> 4 [0,14), leading byte offset >> 4
// [16,30) (unused by swizzled K-major tiles, 1), stride byte offset >> 4 [32,46),
// descriptor version 1 [46,48), base offset 0 [49,52), layout 2 = 128-byte swizzle
// [61,64).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator [4,6) = 1, A and B bf16
// [7,10) = [10,13) = 1, both K-major (bits 15, 16 zero), N >> 3 at [17,23),
// M >> 4 at [24,29).
__device__ __forceinline__ uint32_t f16_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Byte offset of the 16-byte chunk c (0..7) of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// Codes -> floats without integer conversion: nibble j of a word ORed under the
// exponent (150 - 4j) reads as 2^(23-4j) + q exactly, and one packed add removes
// the offset.  Masks and exponents live in registers (one LOP3 per nibble).
struct NibbleConsts {
  uint32_t m0, m1, m2, m3, m4, e150, e146, e142, e138, e134;
};
__device__ __forceinline__ NibbleConsts nibble_consts() {
  NibbleConsts k{0xFu, 0xF0u, 0xF00u, 0xF000u, 0xF0000u,
                 150u << 23, 146u << 23, 142u << 23, 138u << 23, 134u << 23};
  asm volatile("" : "+r"(k.m0), "+r"(k.m1), "+r"(k.m2), "+r"(k.m3), "+r"(k.m4));
  asm volatile("" : "+r"(k.e150), "+r"(k.e146), "+r"(k.e142), "+r"(k.e138), "+r"(k.e134));
  return k;
}
__device__ __forceinline__ float or_and(uint32_t a, uint32_t m, uint32_t e) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(m), "r"(e));
  return __uint_as_float(d);
}
// The 8 codes of w (element j = nibble j) as (q0,q1) (q2,q3) (q4,q5) (q6,q7).
__device__ __forceinline__ void nibbles8(uint32_t w, const NibbleConsts& k, float2 (&q)[4]) {
  const uint32_t w2 = w >> 12;
  q[0] = __fadd2_rn(make_float2(or_and(w, k.m0, k.e150), or_and(w, k.m1, k.e146)),
                    make_float2(-8388608.f, -524288.f));
  q[1] = __fadd2_rn(make_float2(or_and(w, k.m2, k.e142), or_and(w, k.m3, k.e138)),
                    make_float2(-32768.f, -2048.f));
  q[2] = __fadd2_rn(make_float2(or_and(w, k.m4, k.e134), or_and(w2, k.m2, k.e142)),
                    make_float2(-128.f, -32768.f));
  q[3] = __fadd2_rn(make_float2(or_and(w2, k.m3, k.e138), or_and(w2, k.m4, k.e134)),
                    make_float2(-2048.f, -128.f));
}
// Packed bf16 pair (round to nearest even) of two floats: low half = a.
__device__ __forceinline__ uint32_t bf16x2_rn(float a, float b) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(b), "f"(a));
  return d;
}
// One code word's 8 weights w = s*q + b as bf16 hi (= bf16(w)) and lo (= bf16(w - hi)).
__device__ __forceinline__ void dequant8_hilo(uint32_t w, float2 s2, float2 b2,
                                              const NibbleConsts& k, uint4& hi, uint4& lo) {
  float2 q[4];
  nibbles8(w, k, q);
  uint32_t h[4], l[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 v = __ffma2_rn(q[j], s2, b2);
    h[j] = bf16x2_rn(v.x, v.y);
    const float2 hv = make_float2(__uint_as_float(h[j] << 16), __uint_as_float(h[j] & 0xffff0000u));
    const float2 r = __fadd2_rn(v, make_float2(-hv.x, -hv.y));  // exact
    l[j] = bf16x2_rn(r.x, r.y);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// ------------------------------------------------------------------ kernels ---
struct GroupedArgs {
  const uint16_t* act;   // phase 0: x [T, H]; phase 1: h [P, I] (pair_list order)
  const int* unique;     // [u] distinct experts, ascending
  const int* offsets;    // [u + 1]
  const int* pair_list;  // [P] pair ids grouped by expert
  const int* num_unique; // [1]
  const uint32_t *q0, *q1;   // codes: phase 0 gate / up, phase 1 down
  const uint16_t *s0, *b0, *s1, *b1;
  uint16_t* h;           // phase 0 output [P, I] bf16
  float* y;              // phase 1 output [P, H] fp32
  int k, rows, K;        // top-k; weight rows per expert (I or H); K (H or I)
  int H, I;
};

// One launch per phase, one CTA per SM looping over (expert slot, 128-row tile).
template <int PHASE>
__global__ void __launch_bounds__(kGThreads, 1) grouped_kernel(const GroupedArgs a) {
  extern __shared__ __align__(128) unsigned char gsm_raw[];
  __shared__ __align__(8) uint64_t mma_done[2];
  __shared__ uint32_t tmem_base_s;
  // swizzled tiles start at 1024-byte boundaries of the shared address space
  unsigned char* gsm = gsm_raw + ((1024u - (smem_u32(gsm_raw) & 1023u)) & 1023u);
  constexpr int NMAT = PHASE == 0 ? 2 : 1;
  constexpr unsigned kBuf = 2 * NMAT * kGATile + kGBTile;
  constexpr uint32_t kCols = PHASE == 0 ? 2 * kGMaxN : kGMaxN;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_s, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  const int u = *a.num_unique;
  const int mtiles = a.rows / kGM;
  const int nslab = a.K / kGK;
  uint32_t phase_bits = 0;  // completed-phase parity of mma_done[0], [1]
  bool ok = true;
  const NibbleConsts nk = nibble_consts();

  for (int tile = blockIdx.x; tile < u * mtiles && ok; tile += gridDim.x) {
    const int slot = tile / mtiles, m0 = (tile % mtiles) * kGM;
    const int e = a.unique[slot];
    const int p_begin = a.offsets[slot], p_end = a.offsets[slot + 1];
    const size_t wrow0 = (size_t)e * a.rows + m0;  // first weight row of the tile
    for (int n0 = p_begin; n0 < p_end && ok; n0 += kGMaxN) {
      const int n = min(kGMaxN, p_end - n0);
      const int np = (n + 15) & ~15;  // MMA N
      const uint32_t idesc = f16_idesc(kGM, np);
      int issued = 0;  // slabs whose MMAs were issued (in this n-chunk)
      // Per thread: A tasks (matrix, row, half slab of 32 columns) tid and tid + 256
      // (gate+up), B tasks (pair row, 16-byte chunk) tid + 256 i.  Their global data
      // for slab s+1 is loaded while slab s is dequantised and multiplied.
      constexpr int kATasks = NMAT * kGM * 2 / kGThreads;  // 2 or 1
      constexpr int kBTasks = kGMaxN * 8 / kGThreads;      // 8
      uint4 cw[kATasks];
      uint16_t sraw[kATasks], braw[kATasks];
      uint4 xv[kBTasks];
      auto load_slab = [&](int s) {
#pragma unroll
        for (int i = 0; i < kATasks; ++i) {
          const int task = tid + i * kGThreads;
          const int mat = task / (kGM * 2), rr = (task >> 1) % kGM, half = task & 1;
          const uint32_t* q = mat ? a.q1 : a.q0;
          const uint16_t* sp = mat ? a.s1 : a.s0;
          const uint16_t* bp = mat ? a.b1 : a.b0;
          const size_t row = wrow0 + rr;
          cw[i] = __ldg(reinterpret_cast<const uint4*>(q + row * (a.K / 8) + s * 8) + half);
          sraw[i] = __ldg(sp + row * (a.K / 64) + s);
          braw[i] = __ldg(bp + row * (a.K / 64) + s);
        }
#pragma unroll
        for (int i = 0; i < kBTasks; ++i) {
          const int task = tid + i * kGThreads, rr = task >> 3, c = task & 7;
          xv[i] = make_uint4(0u, 0u, 0u, 0u);
          if (rr < n) {
            const int pos = n0 + rr;
            const size_t arow = PHASE == 0 ? (size_t)(a.pair_list[pos] / a.k) : (size_t)pos;
            const uint16_t* src = a.act + arow * a.K + s * kGK + c * 8;
            xv[i] = PHASE == 0 ? __ldg(reinterpret_cast<const uint4*>(src))
                               : __ldcg(reinterpret_cast<const uint4*>(src));
          }
        }
      };
      load_slab(0);
      for (int s = 0; s < nslab && ok; ++s) {
        const int buf = s & 1;
        unsigned char* base = gsm + buf * kBuf;
        if (s >= 2) {  // the MMAs that read this buffer two slabs ago are done
          ok = mbar_wait(&mma_done[buf], (phase_bits >> buf) & 1);
          phase_bits ^= 1u << buf;
          if (!ok) break;
        }
        uint4 ccw[kATasks], cxv[kBTasks];
        uint16_t cs[kATasks], cb[kATasks];
#pragma unroll
        for (int i = 0; i < kATasks; ++i) {
          ccw[i] = cw[i];
          cs[i] = sraw[i];
          cb[i] = braw[i];
        }
#pragma unroll
        for (int i = 0; i < kBTasks; ++i) cxv[i] = xv[i];
        if (s + 1 < nslab) load_slab(s + 1);
        // --- A: dequantised weight slab(s), 128 rows x 64, hi and lo, swizzled ---
#pragma unroll
        for (int i = 0; i < kATasks; ++i) {
          const int task = tid + i * kGThreads;
          const int mat = task / (kGM * 2), rr = (task >> 1) % kGM, half = task & 1;
          const float sc = bf16_bits_to_float(cs[i]), bi = bf16_bits_to_float(cb[i]);
          const float2 s2 = make_float2(sc, sc), b2 = make_float2(bi, bi);
          unsigned char* tileA = base + 2 * mat * kGATile;  // hi tile; lo tile follows
          const uint32_t ws[4] = {ccw[i].x, ccw[i].y, ccw[i].z, ccw[i].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // 16-byte chunk = 8 columns = one code word
            uint4 hi, lo;
            dequant8_hilo(ws[c], s2, b2, nk, hi, lo);
            const uint32_t off = sw128_off(rr, half * 4 + c);
            *reinterpret_cast<uint4*>(tileA + off) = hi;
            *reinterpret_cast<uint4*>(tileA + kGATile + off) = lo;
          }
        }
        // --- B: the activation rows of the slab (zero rows up to np), swizzled ---
        unsigned char* tileB = base + 2 * NMAT * kGATile;
#pragma unroll
        for (int i = 0; i < kBTasks; ++i) {
          const int task = tid + i * kGThreads, rr = task >> 3, c = task & 7;
          if (rr < np) *reinterpret_cast<uint4*>(tileB + sw128_off(rr, c)) = cxv[i];
        }
        fence_proxy_async();  // generic smem writes -> tensor-core reads
        __syncthreads();
        if (tid == 0) {
          tc_fence_after();
          const uint32_t a_addr = smem_u32(base), b_addr = smem_u32(tileB);
#pragma unroll
          for (int kk = 0; kk < kGK / 16; ++kk) {
            const uint64_t bdesc = sw128_desc(b_addr + kk * 32);
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat) {
              const uint32_t a_hi = a_addr + 2 * mat * kGATile + kk * 32;
              tc_mma(tmem + mat * kGMaxN, sw128_desc(a_hi), bdesc, idesc,
                     (s > 0 || kk > 0) ? 1u : 0u);
              tc_mma(tmem + mat * kGMaxN, sw128_desc(a_hi + kGATile), bdesc, idesc, 1u);
            }
          }
          tc_commit(&mma_done[buf]);
        }
        ++issued;
      }
      // all MMAs of the chunk done (the last one or two commits not waited yet)
      for (int s = (issued > 2 ? issued - 2 : 0); s < issued && ok; ++s) {
        const int buf = s & 1;
        ok = mbar_wait(&mma_done[buf], (phase_bits >> buf) & 1);
        phase_bits ^= 1u << buf;
      }
      tc_fence_after();
      // --- epilogue: warp w reads lanes 32 (w % 4).., columns half (w / 4) ---
      if (ok) {
        const int r = 32 * (warp & 3) + lane;  // tile row of this thread
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        for (int c0 = (warp >> 2) * 16; c0 < np; c0 += 32) {
          float d0[16];
          tc_ld16(lane_addr + c0, d0);
          if (PHASE == 0) {
            float d1[16];
            tc_ld16(lane_addr + kGMaxN + c0, d1);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (c0 + j < n) {
                const float g = round_to_bf16(d0[j]), uv = round_to_bf16(d1[j]);
                a.h[(size_t)(n0 + c0 + j) * a.I + m0 + r] =
                    float_to_bf16_bits(g / (1.0f + __expf(-g)) * uv);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c0 + j < n) a.y[(size_t)(n0 + c0 + j) * a.H + m0 + r] = d0[j];
          }
        }
      }
      tc_fence_before();
      __syncthreads();  // accumulators read before the next chunk overwrites them
      tc_fence_after();
    }
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kCols);
}

// out[t][c] = bf16(sum_j w[t,j] * y[pos(t,j)][c]), j ascending, for the pairs the
// route-union kept (pos from pair_list); rows of tokens whose pairs were all left
// out are zero.
__global__ void __launch_bounds__(256) grouped_combine_kernel(
    const float* __restrict__ y, const float* __restrict__ w, const int* __restrict__ pair_list,
    const int* __restrict__ offsets, const int* __restrict__ num_unique, int T, int k, int H,
    uint16_t* __restrict__ out) {
  extern __shared__ int pos_of[];  // [T * k]
  const int P = T * k;
  for (int p = threadIdx.x; p < P; p += blockDim.x) pos_of[p] = -1;
  __syncthreads();
  const int nv = offsets[*num_unique];
  for (int i = threadIdx.x; i < nv; i += blockDim.x) pos_of[pair_list[i]] = i;
  __syncthreads();
  const long long total = (long long)T * H;
  for (long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x; o < total;
       o += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(o / H), c = (int)(o % H);
    float acc = 0.f;
    for (int j = 0; j < k; ++j) {
      const int pos = pos_of[t * k + j];
      if (pos >= 0) acc = fmaf(__ldg(w + t * k + j), __ldcg(y + (size_t)pos * H + c), acc);
    }
    out[o] = float_to_bf16_bits(acc);
  }
}

}  // namespace qeg
