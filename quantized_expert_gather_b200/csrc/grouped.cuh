// Large-window path: the same layer as layer.cuh as grouped GEMMs on the 5th-
// generation tensor cores, for windows with more pairs than the persistent
// kernel holds.
//
// "MoE GatherQMM small-M verify cost" (llms-explorer fact sheet): above a pair
// threshold the pairs are sorted by expert and each expert's rows are applied as
// one matrix product (the sorted grouped path).  Here, after the route-union
// (route_union.cuh) has grouped the pairs by expert:
//
//   grouped_pack_x_kernel   the window's x rows, one per pair, in the order and
//                           layout the tensor cores read (below), with group sums;
//   grouped_gemm_kernel<0, N>  gate+up: per (expert, 128 rows of Wg and of Wu) tile,
//                           G = Wg X^T, U = Wu X^T, h = bf16(silu(bf16 G) * bf16 U),
//                           h written packed for the next launch;
//   grouped_gemm_kernel<1, N>  down: per (expert, 256 rows of Wd) tile, Y = Wd H^T,
//                           fp32 per pair;
// (N, the pairs per MMA chunk, is 32, 64 or 96: wider chunks stream an expert's
// weights fewer times when it has many pairs; with 32 two CTAs fit on an SM, which
// doubles the warps that hide the per-slab latency.)
//   grouped_combine_kernel  out[t] = bf16(sum_j w[t,j] * y[t,j]), j ascending.
//
// The quantisation group (64 columns of K) is the MMA's K slab.  Inside a group
// a weight row is s * q + b, so its dot product with an activation row a splits
// as  sum_c w_c a_c = s * (sum_c q_c a_c) + b * (sum_c a_c).  The tensor cores
// form P = sum_c q_c a_c from bf16 operands: the codes 0..15 are exact bf16
// integers, the activations are bf16 already, each product is exact and the sum
// is fp32.  Every slab's P is read back from tensor memory and s * P + b * X (X
// the activation row's group sum) is added to fp32 registers.  No weight is ever
// rounded; the only per-weight work is turning 4-bit codes into bf16 integers.
//
// Roles in a CTA (one or two CTAs per SM, looping over tiles):
//   warp 8      producer: per stage of two slabs, 16-byte async copies of each
//               weight row's codes (64 bytes) and 4-byte ones of its scales and
//               biases, and 1-D bulk copies of the two packed activation slabs and
//               of their group sums;
//   warp 9      MMA issuer: issues tcgen05.mma (one elected lane of the converged
//               warp) with A (the codes as bf16) in tensor memory and B (the
//               activations) in shared memory;
//   warps 0..7  warps 4m..4m+3 own matrix m of the tile, one weight row per
//               thread (the row's tensor-memory lane).  Per slab they expand the
//               row's codes to bf16 into tensor memory (the MMA's A operand), then
//               read back the previous slab's product and accumulate it.
// Codes expand without conversions: nibble q placed under the bf16 exponent of
// 128 reads as 128 + q, and one packed bf16 FMA takes the 128 off exactly.  That
// puts codes j and j + 4 of a 32-bit code word in one bf16 pair, so K runs in
// the order (0,4,1,5,2,6,3,7) within every 8 columns; the packed activations
// follow the same order.
//
// mxfp4 banks (F = kFmtMx: e2m1 codes, one e8m0 scale 2^(e-127) per 32 columns, no
// bias): a weight e2m1(q) 2^(e-127) is itself exact in bf16, so the expansion writes
// the weights (two byte lookups give 2 e2m1(q) + 12 per code, placed under the bf16
// exponent of 128 as above, and one packed FMA scales and offsets them exactly), and
// a chunk's whole K accumulates in tensor memory, read back once per chunk.
//
// Packed activations (the B operand): [K/64][pcap][64] bf16.  Row = padded pair
// position: expert slot i owns rows padded[i] .. padded[i] + roundup16(count_i)
// (route_union_kernel's padded offsets), with zero rows as padding.  Each 128-byte
// row holds one slab in the K order above, its 16-byte chunk c stored at chunk
// (c ^ (row & 7)): the 128-byte swizzle of a K-major tile whose rows start at
// multiples of 8.  Group sums: [K/64][pcap] fp32.
#pragma once

#include "common.cuh"
#include "layer.cuh"  // kFmtMx, mx_bytes, mx_half_scale: the mxfp4 code and scale lookups

namespace qeg {

constexpr int kGWorkers = 8;                         // worker warps
constexpr int kGThreads = 32 * (kGWorkers + 2);      // + producer warp + MMA warp
constexpr int kGM = 128;                             // weight rows per matrix (MMA M)
constexpr int kGK = 64;                              // K per slab = quantisation group
constexpr int kGSlabsPerStage = 2;
constexpr unsigned kGCodePitch = kGSlabsPerStage * 32 + 16;  // padded: no bank conflicts
constexpr unsigned kGOffB = 2 * kGM * kGCodePitch;           // 20480, a multiple of 1024
constexpr int kGDBufs = 2;   // accumulator buffers
constexpr int kGLag = 1;     // a slab's accumulator is read back after the next slab's A is stored
constexpr int kGABufs = 2;   // A operand buffers

// Per chunk width NMAX (pairs per MMA, a multiple of 32): the shared-memory stage
// [codes | two activation slabs | their sums | scales | biases] and the tensor
// memory map (accumulator of buffer db, matrix m; then the A operand of buffer ab).
template <int NMAX>
struct GCfg {
  static constexpr int kN = NMAX;
  static constexpr int kStages = NMAX <= 32 ? 3 : (NMAX <= 64 ? 5 : 4);
  static constexpr int kCtasPerSm = NMAX <= 32 ? 2 : 1;  // two CTAs share an SM's tensor memory
  static constexpr uint32_t kTmemCols = NMAX <= 32 ? 256 : 512;
  static constexpr unsigned kBTile = NMAX * kGK * 2;
  static constexpr unsigned kOffX = kGOffB + kGSlabsPerStage * kBTile;
  static constexpr unsigned kOffS = kOffX + kGSlabsPerStage * NMAX * 4;
  static constexpr unsigned kOffBias = kOffS + 2 * kGM * kGSlabsPerStage * 2;
  static constexpr unsigned kStageBytes =
      (kOffBias + 2 * kGM * kGSlabsPerStage * 2 + 1023) & ~1023u;
  static constexpr unsigned kSmem = kStages * kStageBytes + 1024;  // + alignment slack
  static_assert(NMAX % 32 == 0 && kBTile % 1024 == 0, "swizzled tiles need 1024-byte bases");
  static_assert(kGDBufs * 2 * NMAX + kGABufs * 2 * 32 <= (int)kTmemCols, "tensor memory map");
  __device__ static __forceinline__ uint32_t col_d(uint32_t db, int m) {
    return (db * 2 + m) * NMAX;
  }
  __device__ static __forceinline__ uint32_t col_a(uint32_t ab, int m) {
    return kGDBufs * 2 * NMAX + (ab * 2 + m) * 32;
  }
};

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
// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16 (both operands bf16).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same, issued by one elected lane of a converged warp: the whole warp runs the
// issuing code, so its operands stay warp-uniform (issue is several times faster
// than from a single divergent thread).
__device__ __forceinline__ void tc_mma_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit_elect(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(
          smem_u32(bar))
      : "memory");
}
// The mbarrier receives one arrival when every MMA this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane (no wait).
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// After tc_wait_ld: ties 16 loaded registers to the wait, so that no use of them
// is scheduled before it.
__device__ __forceinline__ void tc_regs_ready(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}
// 16 consecutive 32-bit columns of this thread's lane <- r (no wait).
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tc_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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

// 4-byte async copy global -> shared (both 4-byte aligned).
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
// 16-byte async copy global -> shared (both 16-byte aligned), bypassing L1.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
// One arrival on `bar` once this thread's earlier cp.async copies have landed
// (counted in the barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// The 8 codes of word w as 4 bf16 pairs (low half q_j, high half q_{j+4}),
// j = 0..3, exact.  one2 = bf16 pair (1, 1), m128 = (-128, -128).
__device__ __forceinline__ void codes_to_bf16(uint32_t w, uint32_t one2, uint32_t m128,
                                              uint32_t* o) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t t = ((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u;  // 128 + q
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(o[j]) : "r"(t), "r"(one2), "r"(m128));
  }
}

// The 8 mxfp4 codes of word w as 4 bf16 pairs of weights e2m1(q) 2^(e-127) (low
// half code j, high half code j + 4), j = 0..3, exact.  s2 = bf16 pair (h, h) and
// c2 = (-140 h, -140 h) for h = 2^(e-128) of the group's scale byte e: the bytes
// q' = 2 e2m1(q) + 12 read as 128 + q' under the bf16 exponent of 128, and
// (128 + q') h - 140 h = 2 e2m1(q) h.
__device__ __forceinline__ void mx_codes_to_bf16(uint32_t w, uint32_t s2, uint32_t c2,
                                                 uint32_t* o) {
  const uint32_t lo = mx_bytes(w), hi = mx_bytes(w >> 16);  // codes 0..3, 4..7
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // bytes (lo[j], 0, hi[j], 0): selectors j and 4 + j, the others the sign fill of a
    // byte below 128
    const uint32_t sel = (uint32_t)j | ((8u | j) << 4) | ((4u + j) << 8) | ((12u + j) << 12);
    const uint32_t t = prmt_sign(lo, hi, sel) | 0x43004300u;  // 128 + q'
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(o[j]) : "r"(t), "r"(s2), "r"(c2));
  }
}
// The bf16 pairs (h, h) and (-140 h, -140 h), h = 2^(e - 128), for an e8m0 byte e.
__device__ __forceinline__ void mx_scale_pairs(uint32_t e, uint32_t& s2, uint32_t& c2) {
  const float h = mx_half_scale(e);
  const uint32_t hb = float_to_bf16_bits(h), cb = float_to_bf16_bits(-140.0f * h);
  s2 = hb | (hb << 16);
  c2 = cb | (cb << 16);
}

// --------------------------------------------------------------- packing ---
// Packed x: for every padded pair position of every expert slot, the pair's token
// row of x (zero for padding) and its group sums.  One block per slot (looping).
__global__ void __launch_bounds__(256) grouped_pack_x_kernel(
    const uint16_t* __restrict__ x, const int* __restrict__ pair_list,
    const int* __restrict__ offsets, const int* __restrict__ padded,
    const int* __restrict__ num_unique, int k, int H, int pcap, uint16_t* __restrict__ xp,
    float* __restrict__ xs) {
  const int u = *num_unique;
  const int nslab = H / kGK;
  // blocks (slot, y) share a slot's units in strides of gridDim.y * blockDim.x, each
  // thread with kPackBatch loads in flight before the first is used
  constexpr int kPackBatch = 4;
  const int step = gridDim.y * blockDim.x;
  for (int slot = blockIdx.x; slot < u; slot += gridDim.x) {
    const int p0 = offsets[slot], cnt = offsets[slot + 1] - p0;
    const int np = (cnt + 15) & ~15;
    const int base = padded[slot];
    const int units = np * nslab * 8;  // a multiple of 128: whole warps stay together
    for (int u0 = blockIdx.y * blockDim.x + threadIdx.x; u0 < units; u0 += kPackBatch * step) {
      uint4 v[kPackBatch];
#pragma unroll
      for (int i = 0; i < kPackBatch; ++i) {
        const int unit = u0 + i * step;
        const int rest = unit >> 3, n = rest / nslab;
        v[i] = make_uint4(0u, 0u, 0u, 0u);
        if (unit < units && n < cnt) {
          const int c = unit & 7, g = rest % nslab;
          const int t = pair_list[p0 + n] / k;
          v[i] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H + g * kGK + c * 8));
        }
      }
#pragma unroll
      for (int i = 0; i < kPackBatch; ++i) {
        const int unit = u0 + i * step;
        if (unit < units) {  // uniform over the warp (units and step are multiples of 32)
          const int c = unit & 7, rest = unit >> 3;
          const int g = rest % nslab, n = rest / nslab;
          float s = ((bf16_lo(v[i].x) + bf16_hi(v[i].x)) + (bf16_lo(v[i].y) + bf16_hi(v[i].y))) +
                    ((bf16_lo(v[i].z) + bf16_hi(v[i].z)) + (bf16_lo(v[i].w) + bf16_hi(v[i].w)));
          s += __shfl_xor_sync(kFull, s, 1);
          s += __shfl_xor_sync(kFull, s, 2);
          s += __shfl_xor_sync(kFull, s, 4);
          uint4 o;  // K order (0,4,1,5,2,6,3,7)
          o.x = prmt(v[i].x, v[i].z, 0x5410u);
          o.y = prmt(v[i].x, v[i].z, 0x7632u);
          o.z = prmt(v[i].y, v[i].w, 0x5410u);
          o.w = prmt(v[i].y, v[i].w, 0x7632u);
          const int pos = base + n;
          *reinterpret_cast<uint4*>(xp + ((size_t)g * pcap + pos) * kGK + ((c ^ (pos & 7)) * 8)) = o;
          if (c == 0) xs[(size_t)g * pcap + pos] = s;
        }
      }
    }
  }
}

// ------------------------------------------------------------------ GEMMs ---
struct GroupedArgs {
  const uint16_t* bp;    // packed activations [K/64][pcap][64] (x or h)
  const float* bs;       // their group sums [K/64][pcap]
  const int* unique;     // [u] distinct experts, ascending
  const int* offsets;    // [u + 1]
  const int* padded;     // [u + 1] padded row offsets of the packed layout
  const int* num_unique; // [1]
  const uint32_t* q[2];  // codes of matrix 0 / 1 of a tile
  const uint16_t* s[2];  // scales (mxfp4: the e8m0 bytes)
  const uint16_t* b[2];  // biases (mxfp4: none)
  int roff[2];           // row offset of matrix m inside the tile (0/0 or 0/128)
  uint16_t* hp;          // phase 0: packed h [I/64][pcap][64]
  float* hs;             // phase 0: h group sums [I/64][pcap]
  float* y;              // phase 1: [P, H] fp32 in pair_list order
  int rows, K, mrows;    // weight rows per expert; K; weight rows per tile
  int pcap, H;
};

template <int PHASE, int NMAX, int F = kFmtAffine>
__global__ void __launch_bounds__(kGThreads, GCfg<NMAX>::kCtasPerSm)
    grouped_gemm_kernel(const __grid_constant__ GroupedArgs a) {
  using C = GCfg<NMAX>;
  extern __shared__ __align__(128) unsigned char gsm_raw[];
  __shared__ __align__(8) uint64_t full[C::kStages], empty[C::kStages];
  __shared__ __align__(8) uint64_t a_full[kGABufs], d_full[kGDBufs], d_free[kGDBufs];
  __shared__ __align__(8) uint64_t c_full[kGDBufs];  // mxfp4: a chunk's product complete
  __shared__ uint32_t tmem_base_s;
  __shared__ float red[2][2][C::kN / 2];
  // swizzled tiles start at 1024-byte boundaries of the shared address space
  unsigned char* gsm = gsm_raw + ((1024u - (smem_u32(gsm_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1 + 32);          // expect_tx + one cp.async arrival per lane
      mbar_init(&empty[i], kGWorkers + 1);  // worker warps + the MMA commit
    }
    for (int i = 0; i < kGABufs; ++i) mbar_init(&a_full[i], kGWorkers);
    for (int i = 0; i < kGDBufs; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_free[i], kGWorkers);
      mbar_init(&c_full[i], 1);
    }
    fence_barrier_init();
  }
  if (warp == kGWorkers + 1) {
    tmem_alloc(&tmem_base_s, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(kFull, tmem_base_s, 0);  // warp-uniform

  const int u = *a.num_unique;
  const int mtiles = a.rows / a.mrows;
  const int nslab = a.K / kGK;
  const int ntiles = u * mtiles;
  bool ok = true;
  uint32_t sc = 0;  // stages started (the same sequence in every role)
  uint32_t gs = 0;  // slabs started

  if (warp == kGWorkers) {
    // ------------------------------------------------------------ producer ---
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int slot = tile / mtiles, m0 = (tile % mtiles) * a.mrows;
      const int e = a.unique[slot];
      const int cnt = a.offsets[slot + 1] - a.offsets[slot];
      const int pp0 = a.padded[slot];
      for (int c0 = 0; c0 < cnt && ok; c0 += C::kN) {
        const int np = (min(C::kN, cnt - c0) + 15) & ~15;
        for (int j0 = 0; j0 < nslab && ok; j0 += kGSlabsPerStage) {
          const int st = sc % C::kStages;
          const uint32_t round = sc / C::kStages;
          if (lane == 0) {
            if (round > 0) ok = mbar_wait(&empty[st], (round - 1) & 1);
            if (ok)
              mbar_arrive_expect_tx(&full[st], kGSlabsPerStage * np * (kGK * 2 + 4));
          }
          ok = __shfl_sync(kFull, ok, 0);
          if (!ok) break;
          unsigned char* stg = gsm + st * C::kStageBytes;
          // codes: 16 bytes per lane, four lanes per row (64 bytes = two slabs)
#pragma unroll 8
          for (int i = 0; i < 2 * kGM * kGSlabsPerStage * 2 / 32; ++i) {
            const int ci = lane + 32 * i, rr = ci >> 2, c = ci & 3;
            const int m = rr / kGM, r = rr % kGM;
            const size_t row = (size_t)e * a.rows + m0 + a.roff[m] + r;
            cp_async16(stg + rr * kGCodePitch + c * 16, a.q[m] + row * (a.K / 8) + j0 * 8 + c * 4);
          }
          // scales and biases of the two slabs: 4 bytes per row each
#pragma unroll
          for (int i = 0; i < 2 * kGM / 32; ++i) {
            const int rr = lane + 32 * i, m = rr / kGM, r = rr % kGM;
            const size_t row = (size_t)e * a.rows + m0 + a.roff[m] + r;
            if constexpr (F == kFmtMx) {  // the stage's four e8m0 bytes; no biases
              cp_async4(stg + C::kOffS + rr * 4,
                        reinterpret_cast<const unsigned char*>(a.s[m]) + row * (a.K / 32) + 2 * j0);
            } else {
              cp_async4(stg + C::kOffS + rr * 4, a.s[m] + row * (a.K / kGK) + j0);
              cp_async4(stg + C::kOffBias + rr * 4, a.b[m] + row * (a.K / kGK) + j0);
            }
          }
          if (lane == 0) {
#pragma unroll
            for (int jj = 0; jj < kGSlabsPerStage; ++jj) {
              const size_t prow = (size_t)(j0 + jj) * a.pcap + pp0 + c0;
              bulk_g2s(stg + kGOffB + jj * C::kBTile, a.bp + prow * kGK, np * kGK * 2, &full[st]);
              bulk_g2s(stg + C::kOffX + jj * C::kN * 4, a.bs + prow, np * 4, &full[st]);
            }
          }
          cp_async_arrive_noinc(&full[st]);
          ++sc;
        }
      }
    }
    // leave no copy in flight: every stage issued has landed (at once when all went well)
    if (lane == 0)
      for (uint32_t i = sc > (uint32_t)C::kStages ? sc - C::kStages : 0; i < sc; ++i)
        mbar_wait(&full[i % C::kStages], (i / C::kStages) & 1);
  } else if (warp == kGWorkers + 1) {
    // ---------------------------------------------------------- MMA issuer ---
    // The whole warp runs this loop (operands warp-uniform); one elected lane issues.
    uint32_t issued = 0;  // slabs whose MMAs were issued
    uint32_t tcn = 0;     // chunks started (mxfp4)
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int slot = tile / mtiles;
      const int cnt = a.offsets[slot + 1] - a.offsets[slot];
      for (int c0 = 0; c0 < cnt && ok; c0 += C::kN) {
        const int np = (min(C::kN, cnt - c0) + 15) & ~15;
        const uint32_t idesc = f16_idesc(kGM, np);
        if constexpr (F == kFmtMx) {
          // The weights are exact in bf16: the chunk's whole K accumulates in
          // accumulator buffer tcn % 2, read back once (c_full); d_full[slab % 2] only
          // says that a slab's MMAs are done, so that its A buffer may be rewritten.
          const uint32_t db = tcn % kGDBufs;
          if (tcn >= (uint32_t)kGDBufs)
            ok = __all_sync(kFull, mbar_wait(&d_free[db], (tcn / kGDBufs - 1) & 1));
          bool first = true;
          for (int j0 = 0; j0 < nslab && ok; j0 += kGSlabsPerStage, ++sc) {
            const int st = sc % C::kStages;
            ok = __all_sync(kFull, mbar_wait(&full[st], (sc / C::kStages) & 1));
            const uint32_t bbase = smem_u32(gsm + st * C::kStageBytes + kGOffB);
            for (int jj = 0; jj < kGSlabsPerStage && ok; ++jj, ++gs) {
              const uint32_t ab = gs % kGABufs;
              ok = __all_sync(kFull, mbar_wait(&a_full[ab], (gs / kGABufs) & 1));
              if (!ok) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < kGK / 16; ++kk) {
                const uint64_t bdesc = sw128_desc(bbase + jj * C::kBTile + kk * 32);
#pragma unroll
                for (int m = 0; m < 2; ++m)
                  tc_mma_ts_elect(tmem + C::col_d(db, m), tmem + C::col_a(ab, m) + kk * 8, bdesc,
                                  idesc, (first && kk == 0) ? 0u : 1u);
              }
              first = false;
              tc_commit_elect(&d_full[ab]);
              if (jj == kGSlabsPerStage - 1) tc_commit_elect(&empty[st]);
              issued = gs + 1;
            }
          }
          if (ok) tc_commit_elect(&c_full[db]);
          ++tcn;
        } else {
          for (int j0 = 0; j0 < nslab && ok; j0 += kGSlabsPerStage, ++sc) {
            const int st = sc % C::kStages;
            const uint32_t round = sc / C::kStages;
            ok = __all_sync(kFull, mbar_wait(&full[st], round & 1));
            const uint32_t bbase = smem_u32(gsm + st * C::kStageBytes + kGOffB);
            for (int jj = 0; jj < kGSlabsPerStage && ok; ++jj, ++gs) {
              const uint32_t ab = gs % kGABufs, db = gs % kGDBufs;
              bool w = mbar_wait(&a_full[ab], (gs / kGABufs) & 1);
              if (w && gs >= (uint32_t)kGDBufs) w = mbar_wait(&d_free[db], (gs / kGDBufs - 1) & 1);
              ok = __all_sync(kFull, w);
              if (!ok) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < kGK / 16; ++kk) {
                const uint64_t bdesc = sw128_desc(bbase + jj * C::kBTile + kk * 32);
#pragma unroll
                for (int m = 0; m < 2; ++m)
                  tc_mma_ts_elect(tmem + C::col_d(db, m), tmem + C::col_a(ab, m) + kk * 8, bdesc,
                                  idesc, kk > 0 ? 1u : 0u);
              }
              tc_commit_elect(&d_full[db]);
              if (jj == kGSlabsPerStage - 1) tc_commit_elect(&empty[st]);
              issued = gs + 1;
            }
          }
        }
      }
    }
    // no MMA may run past the deallocation below (at once when all went well)
    if (issued > 0) mbar_wait(&d_full[(issued - 1) % kGDBufs], ((issued - 1) / kGDBufs) & 1);
  } else {
    // ------------------------------------------------------------- workers ---
    const int m = warp >> 2, qd = warp & 3, r = 32 * qd + lane;
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    const uint32_t one2 = 0x3F803F80u, m128 = 0xC300C300u;  // bf16 pairs (1, 1), (-128, -128)
    float2 acc[C::kN / 2];

    // wait until the MMAs of slab gp are done (its accumulator is ready and the A
    // buffer it read is free)
    auto wait_slab = [&](uint32_t gp) {
      ok = __all_sync(kFull, ok && mbar_wait(&d_full[gp % kGDBufs], (gp / kGDBufs) & 1));
    };
    // add the product of slab gp (stage st, place jj in the stage) to acc; its
    // MMAs are known to be done
    auto readout = [&](uint32_t gp, int st, int jj, int ng) {
      const uint32_t ab = gp % kGDBufs;
      tc_fence_after();
      const unsigned char* stg = gsm + st * C::kStageBytes;
      float sv = 1.0f, bv = 0.0f;  // mxfp4: the weights carry their scale, no bias
      if constexpr (F != kFmtMx) {
        sv = bf16_bits_to_float(
            *reinterpret_cast<const uint16_t*>(stg + C::kOffS + (m * kGM + r) * 4 + jj * 2));
        bv = bf16_bits_to_float(
            *reinterpret_cast<const uint16_t*>(stg + C::kOffBias + (m * kGM + r) * 4 + jj * 2));
      }
      const float2 s2 = make_float2(sv, sv), b2 = make_float2(bv, bv);
      const float4* X = reinterpret_cast<const float4*>(stg + C::kOffX + jj * C::kN * 4);
      const uint32_t dcol = tmem + C::col_d(ab, m) + lane_base;
      // kRd columns per tensor-memory wait (16 where registers are scarce)
      constexpr int kRd = C::kN == 64 ? 32 : 16, kRg = kRd / 16;
#pragma unroll
      for (int c2 = 0; c2 < C::kN / kRd; ++c2) {
        if (kRg * c2 < ng) {
          uint32_t pr[kRd];
          tc_ld16(dcol + c2 * kRd, pr);
          if constexpr (kRg == 2) {
            if (2 * c2 + 1 < ng) tc_ld16(dcol + c2 * kRd + 16, pr + 16);
          }
          tc_wait_ld();
#pragma unroll
          for (int h = 0; h < kRg; ++h) {
            const int cg = kRg * c2 + h;
            if (cg < ng) {
              tc_regs_ready(pr + 16 * h);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 xv = X[cg * 4 + i];
                const int o = cg * 8 + 2 * i;
                const uint32_t* pp = pr + 16 * h + 4 * i;
                acc[o] = __ffma2_rn(make_float2(__uint_as_float(pp[0]), __uint_as_float(pp[1])),
                                    s2, acc[o]);
                acc[o + 1] = __ffma2_rn(
                    make_float2(__uint_as_float(pp[2]), __uint_as_float(pp[3])), s2, acc[o + 1]);
                if constexpr (F != kFmtMx) {
                  acc[o] = __ffma2_rn(make_float2(xv.x, xv.y), b2, acc[o]);
                  acc[o + 1] = __ffma2_rn(make_float2(xv.z, xv.w), b2, acc[o + 1]);
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&d_free[ab]);
        if (jj == kGSlabsPerStage - 1) mbar_arrive(&empty[st]);
      }
    };

    // mxfp4: acc = the chunk's product in accumulator buffer db (its MMAs are known to
    // be done), then the buffer is free again
    auto read_chunk = [&](uint32_t db, int ng) {
      tc_fence_after();
      const uint32_t dcol = tmem + C::col_d(db, m) + lane_base;
#pragma unroll
      for (int cg = 0; cg < C::kN / 16; ++cg) {
        if (cg < ng) {
          uint32_t pr[16];
          tc_ld16(dcol + cg * 16, pr);
          tc_wait_ld();
          tc_regs_ready(pr);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[cg * 8 + i] = make_float2(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_free[db]);
    };
    uint32_t tcn = 0;  // chunks finished (mxfp4)

    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int slot = tile / mtiles, m0 = (tile % mtiles) * a.mrows;
      const int p0 = a.offsets[slot], cnt = a.offsets[slot + 1] - p0;
      const int pp0 = a.padded[slot];
      for (int c0 = 0; c0 < cnt && ok; c0 += C::kN) {
        const int n = min(C::kN, cnt - c0), np = (n + 15) & ~15, ng = np / 16;
#pragma unroll
        for (int i = 0; i < C::kN / 2; ++i) acc[i] = make_float2(0.f, 0.f);
        const uint32_t gs0 = gs, sc0 = sc;  // first slab and stage of the chunk
        // slab g of this chunk: stage (sc0 + (g - gs0) / 2) % C::kStages, place (g - gs0) & 1
        auto read_slab = [&](uint32_t g) {
          const uint32_t jl = g - gs0;
          readout(g, (int)((sc0 + jl / kGSlabsPerStage) % C::kStages), (int)(jl % kGSlabsPerStage), ng);
        };
        for (int j0 = 0; j0 < nslab && ok; j0 += kGSlabsPerStage, ++sc) {
          const int st = sc % C::kStages;
          const uint32_t round = sc / C::kStages;
          ok = __all_sync(kFull, mbar_wait(&full[st], round & 1));
          if (!ok) break;
          const unsigned char* stg = gsm + st * C::kStageBytes;
          for (int jj = 0; jj < kGSlabsPerStage && ok; ++jj, ++gs) {
            const uint32_t ab = gs % kGABufs;
            // the MMAs that read this A buffer (slab gs - 2) are done
            if (gs >= (uint32_t)kGABufs) wait_slab(gs - kGABufs);
            if (!ok) break;
            tc_fence_after();  // the A buffer's earlier reads are done before these writes
            // this row's codes of the slab -> bf16 integers -> the A operand
            const uint4* crow =
                reinterpret_cast<const uint4*>(stg + (m * kGM + r) * kGCodePitch + jj * 32);
            const uint32_t acol = tmem + C::col_a(ab, m) + lane_base;
#pragma unroll
            for (int hw = 0; hw < 2; ++hw) {  // 32 codes (16 columns) at a time
              const uint4 wv = crow[hw];
              uint32_t av[16];
              if constexpr (F == kFmtMx) {  // one e8m0 group: this slab's byte hw
                uint32_t s2, c2;
                mx_scale_pairs(stg[C::kOffS + (m * kGM + r) * 4 + jj * 2 + hw], s2, c2);
                mx_codes_to_bf16(wv.x, s2, c2, av + 0);
                mx_codes_to_bf16(wv.y, s2, c2, av + 4);
                mx_codes_to_bf16(wv.z, s2, c2, av + 8);
                mx_codes_to_bf16(wv.w, s2, c2, av + 12);
              } else {
                codes_to_bf16(wv.x, one2, m128, av + 0);
                codes_to_bf16(wv.y, one2, m128, av + 4);
                codes_to_bf16(wv.z, one2, m128, av + 8);
                codes_to_bf16(wv.w, one2, m128, av + 12);
              }
              tc_st16(acol + 16 * hw, av);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[ab]);
            if constexpr (F == kFmtMx) {
              // the stage's codes and scale bytes are read: release it (the MMA warp's
              // commit is the other arrival)
              if (jj == kGSlabsPerStage - 1 && lane == 0) mbar_arrive(&empty[st]);
            } else if (gs >= gs0 + kGLag) {
              wait_slab(gs - kGLag);
              if (ok) read_slab(gs - kGLag);
            }
          }
        }
        if (!ok) break;
        if constexpr (F == kFmtMx) {
          // the chunk's whole product, accumulated over K in tensor memory, read once
          const uint32_t db = tcn % kGDBufs;
          ok = __all_sync(kFull, mbar_wait(&c_full[db], (tcn / kGDBufs) & 1));
          if (!ok) break;
          read_chunk(db, ng);
          ++tcn;
        } else {
          // the chunk's last kGLag slabs
          for (uint32_t g = gs >= gs0 + kGLag ? gs - kGLag : gs0; g < gs && ok; ++g) {
            wait_slab(g);
            if (ok) read_slab(g);
          }
        }
        if (!ok) break;

        if (PHASE == 0) {
          // ---- h = bf16(silu(bf16 g) * bf16 u); matrix 0 holds g, matrix 1 u.  The
          // two warps of a lane quarter swap halves through tensor memory (buffer 0's
          // accumulator columns): no MMA runs now, the next one waits for every
          // warp's next A operand.
          const int irow = m0 + r;  // this thread's row of h's width I
          const int gI = irow / kGK, ci = irow % kGK;
          const int pin = (ci & ~7) + 2 * (ci & 3) + ((ci >> 2) & 1);  // K order position
          constexpr int kHalf = C::kN / 2;  // pairs finished by each matrix's warps
#pragma unroll
          for (int hh = 0; hh < kHalf / 16; ++hh) {
            // 16 pairs per round: this thread finishes pairs kHalf m + 16hh + i
            uint32_t ex[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 v = m == 0 ? acc[kHalf / 2 + 8 * hh + i] : acc[8 * hh + i];
              ex[2 * i] = __float_as_uint(v.x);
              ex[2 * i + 1] = __float_as_uint(v.y);
            }
            // each warp writes only its own matrix's columns (its partner may still be
            // reading the other matrix's): matrix 0 gives g of pairs kHalf + 16hh.. at
            // its columns kHalf + 16hh.., matrix 1 gives u of pairs 16hh.. at its
            // columns 16hh..
            const uint32_t give =
                tmem + C::col_d(0, m) + (m == 0 ? kHalf : 0) + 16 * hh + lane_base;
            const uint32_t take =
                tmem + C::col_d(0, 1 - m) + (m == 0 ? 0 : kHalf) + 16 * hh + lane_base;
            tc_st16(give, ex);
            tc_wait_st();
            tc_fence_before();
            named_barrier(1 + qd, 64);
            tc_fence_after();
            uint32_t ot[16];
            tc_ld16(take, ot);
            tc_wait_ld();
            tc_regs_ready(ot);
            tc_fence_before();
            float hv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 mine = m == 0 ? acc[8 * hh + i / 2] : acc[kHalf / 2 + 8 * hh + i / 2];
              const float own = (i & 1) ? mine.y : mine.x;
              const float oth = __uint_as_float(ot[i]);
              const float g = round_to_bf16(m == 0 ? own : oth);
              const float uu = round_to_bf16(m == 0 ? oth : own);
              const uint16_t hb = float_to_bf16_bits(g / (1.0f + __expf(-g)) * uu);
              hv[i] = bf16_bits_to_float(hb);
              const int nn = kHalf * m + 16 * hh + i;
              if (nn < np) {
                const int pos = pp0 + c0 + nn;
                a.hp[((size_t)gI * a.pcap + pos) * kGK + (((pin >> 3) ^ (pos & 7)) << 3) +
                     (pin & 7)] = hb;
              }
            }
            // group sums of h: over this warp's 32 rows (even lanes end with one
            // pair's sum each), then over the group's two warps
            int vid;
            const float part = warp_reduce_scatter<16>(hv, lane, vid);
            if ((qd & 1) && !(lane & 1)) red[m][qd >> 1][16 * hh + vid] = part;
            named_barrier(5 + 2 * m + (qd >> 1), 64);
            if (!(qd & 1) && !(lane & 1)) {
              const int nn = kHalf * m + 16 * hh + vid;
              if (nn < np)
                a.hs[(size_t)gI * a.pcap + pp0 + c0 + nn] = part + red[m][qd >> 1][16 * hh + vid];
            }
            named_barrier(5 + 2 * m + (qd >> 1), 64);
          }
        } else {
          // ---- y rows of the chunk's pairs (pair_list order), fp32
          float* yo = a.y + (size_t)(p0 + c0) * a.H + m0 + a.roff[m] + r;
#pragma unroll
          for (int i = 0; i < C::kN; ++i)
            if (i < n) yo[(size_t)i * a.H] = (i & 1) ? acc[i / 2].y : acc[i / 2].x;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kGWorkers + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// out[t][c] = bf16(sum_j w[t,j] * y[pos(t,j)][c]), j ascending, for the pairs the
// route-union kept (pos from pair_list); rows of tokens whose pairs were all left
// out are zero.  Bound by reading y: launched with two 512-thread CTAs per SM so
// that enough loads are in flight.
constexpr int kGCombineThreads = 512;
__global__ void __launch_bounds__(kGCombineThreads) grouped_combine_kernel(
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
  // four consecutive columns per thread (H is a multiple of 4): one 16-byte load of y
  // per pair; each column's sum runs over j in ascending order as a chain of fmaf
  const int H4 = H / 4;
  const long long total = (long long)T * H4;
  for (long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x; o < total;
       o += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(o / H4), c4 = (int)(o % H4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int pos = pos_of[t * k + j];
      if (pos >= 0) {
        const float wj = __ldg(w + t * k + j);
        const float4 yv = __ldcg(reinterpret_cast<const float4*>(y + (size_t)pos * H) + c4);
        acc.x = fmaf(wj, yv.x, acc.x);
        acc.y = fmaf(wj, yv.y, acc.y);
        acc.z = fmaf(wj, yv.z, acc.z);
        acc.w = fmaf(wj, yv.w, acc.w);
      }
    }
    uint2 ob;
    ob.x = (uint32_t)float_to_bf16_bits(acc.x) | ((uint32_t)float_to_bf16_bits(acc.y) << 16);
    ob.y = (uint32_t)float_to_bf16_bits(acc.z) | ((uint32_t)float_to_bf16_bits(acc.w) << 16);
    reinterpret_cast<uint2*>(out + (size_t)t * H)[c4] = ob;
  }
}

}  // namespace qeg
