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
//                           layout the tensor cores read (below);
//   grouped_gemm_kernel<0, N>  gate+up: per (expert, 128 rows of Wg and of Wu) tile,
//                           G = Wg X^T, U = Wu X^T, h = bf16(silu(bf16 G) * bf16 U),
//                           h written packed for the next launch;
//   grouped_gemm_kernel<1, N>  down: per (expert, 256 rows of Wd) tile, Y = Wd H^T,
//                           fp32 per pair;
// (N, the most pairs per MMA chunk, is 32, 64 or 96: wider chunks stream an
// expert's weights fewer times when it has many pairs, narrower ones leave shared
// memory for a deeper copy ring.)
//   grouped_combine_kernel  out[t] = bf16(sum_j w[t,j] * y[t,j]), j ascending.
//
// Arithmetic.  Each weight is dequantised once, w = bf16(s * q + b) (one fused
// multiply-add on bf16 pairs, a single rounding of the exact s*q+b), the weight
// rows of a tile become the MMA's A operand in shared memory, the packed bf16
// activation rows its B operand, and the tensor cores accumulate the whole K of
// the tile in fp32 in tensor memory.  The product is read once per tile.
//
// Roles in a CTA (one CTA per SM, looping over tiles):
//   warps 0..7   dequantisers: warps 4m..4m+3 own matrix m of the tile, one weight
//                row per thread.  Per K slab of 64 columns (one quantisation group)
//                a thread turns its row's 64 codes into bf16 weights and stores
//                them in the A buffer (two buffers) in the MMA's layout;
//   warps 8..11  epilogue: read a finished tile's accumulators (two buffers) from
//                tensor memory, one row per thread, and write h (gate+up) or y
//                (down);
//   warp 12      producer: per stage of two slabs, 16-byte async copies of each
//                weight row's codes (64 bytes) and 4-byte ones of its scales and
//                biases, and 1-D bulk copies of the two packed activation slabs;
//   warp 13      MMA issuer: tcgen05.mma (one elected lane of the converged
//                warp) with A and B in shared memory, D in tensor memory.
// Codes expand without conversions: nibble q placed under the bf16 exponent of
// 128 reads as 128 + q, and one packed bf16 FMA takes the 128 off exactly.  That
// puts codes j and j + 4 of a 32-bit code word in one bf16 pair, so K runs in
// the order (0,4,1,5,2,6,3,7) within every 8 columns; the packed activations
// follow the same order.
//
// Operand layout (A and B alike): K-major rows of 128 bytes (one slab), 16-byte
// chunk c of row p stored at chunk (c ^ (p & 7)), 8-row groups 1024 bytes apart:
// the 128-byte swizzle, tiles based at 1024-byte boundaries.  Packed activations
// in global memory: [K/64][pcap][64] bf16, row = padded pair position (expert slot
// i owns rows padded[i] .. padded[i] + roundup16(count_i), route_union_kernel's
// padded offsets; padding rows are zero), swizzled by the global row index.
#pragma once

#include "common.cuh"

namespace qeg {

constexpr int kGDeq = 8;                               // dequantising warps
constexpr int kGEpi = 4;                               // epilogue warps
constexpr int kGProducer = kGDeq + kGEpi;              // warp 12
constexpr int kGMmaWarp = kGProducer + 1;              // warp 13
constexpr int kGThreads = 32 * (kGMmaWarp + 1);        // 448
constexpr int kGM = 128;                               // weight rows per matrix (MMA M)
constexpr int kGK = 64;                                // K per slab = quantisation group
constexpr int kGSlabsPerStage = 2;
constexpr unsigned kGCodePitch = kGSlabsPerStage * 32 + 16;  // padded: no bank conflicts
constexpr unsigned kGCodeBytes = 2 * kGM * kGCodePitch;      // 20480
constexpr unsigned kGSbBytes = 2 * kGM * kGSlabsPerStage * 2;  // scales (or biases) of a stage
constexpr int kGABufs = 2;                             // A operand buffers
constexpr unsigned kGATile = kGM * kGK * 2;            // one matrix's slab of A: 16 KB
constexpr unsigned kGABytes = 2 * kGATile;             // one A buffer (both matrices)
constexpr int kGAccBufs = 2;                           // accumulator buffers
constexpr unsigned kGSmemBudget = 230400;              // dynamic shared memory planned for

// Per chunk width NMAX (most pairs per MMA, a multiple of 32): the shared-memory
// stage [codes | scales | biases | two activation slabs], the ring depth and the
// tensor-memory map (accumulator buffer db, matrix m at columns (2 db + m) NMAX).
template <int NMAX>
struct GCfg {
  static constexpr int kN = NMAX;
  static constexpr unsigned kBTile = NMAX * kGK * 2;
  static constexpr unsigned kOffS = kGCodeBytes;
  static constexpr unsigned kOffBias = kOffS + kGSbBytes;
  static constexpr unsigned kOffB = kOffBias + kGSbBytes;  // 22528, a multiple of 1024
  static constexpr unsigned kStageBytes = kOffB + kGSlabsPerStage * kBTile;
  static constexpr unsigned kRing = kGSmemBudget - 1024 - kGABufs * kGABytes;
  static constexpr int kStages = (int)(kRing / kStageBytes) > 6 ? 6 : (int)(kRing / kStageBytes);
  static constexpr unsigned kSmem = kGABufs * kGABytes + kStages * kStageBytes + 1024;
  static constexpr uint32_t kTmemCols =
      kGAccBufs * 2 * NMAX <= 128 ? 128 : (kGAccBufs * 2 * NMAX <= 256 ? 256 : 512);
  static_assert(NMAX % 32 == 0 && kBTile % 1024 == 0 && kOffB % 1024 == 0,
                "swizzled tiles need 1024-byte bases");
  static_assert(kStages >= 2 && kSmem <= kGSmemBudget, "shared-memory plan");
  static_assert(kGAccBufs * 2 * NMAX <= 512, "tensor memory map");
  __device__ static __forceinline__ uint32_t col_d(uint32_t db, int m) {
    return (db * 2 + m) * NMAX;
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
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (both operands bf16),
// issued by one elected lane of a converged warp: the whole warp runs the issuing
// code, so its operands stay warp-uniform (issue is several times faster than from
// a single divergent thread).
__device__ __forceinline__ void tc_mma_ss_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
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

// bf16 pair fused multiply-add, one rounding: a * b + c.
__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// The 8 codes of word w as 4 bf16 pairs of dequantised weights bf16(s q + b)
// (low half code j, high half code j + 4), j = 0..3.  one2 = bf16 pair (1, 1),
// m128 = (-128, -128), s2 / b2 = the group's scale / bias in both halves.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t one2, uint32_t m128,
                                              uint32_t s2, uint32_t b2) {
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t t = ((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u;  // 128 + q, exact
    o[j] = bf16x2_fma(bf16x2_fma(t, one2, m128), s2, b2);             // q exact, then s q + b
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// --------------------------------------------------------------- packing ---
// Packed x: for every padded pair position of every expert slot, the pair's token
// row of x (zero for padding).  One block per slot (looping).
__global__ void __launch_bounds__(256) grouped_pack_x_kernel(
    const uint16_t* __restrict__ x, const int* __restrict__ pair_list,
    const int* __restrict__ offsets, const int* __restrict__ padded,
    const int* __restrict__ num_unique, int k, int H, int pcap, uint16_t* __restrict__ xp) {
  const int u = *num_unique;
  const int nslab = H / kGK;
  for (int slot = blockIdx.x; slot < u; slot += gridDim.x) {
    const int p0 = offsets[slot], cnt = offsets[slot + 1] - p0;
    const int np = (cnt + 15) & ~15;
    const int base = padded[slot];
    const int units = np * nslab * 8;
    for (int unit = threadIdx.x; unit < units; unit += blockDim.x) {
      const int c = unit & 7, rest = unit >> 3;
      const int g = rest % nslab, n = rest / nslab;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (n < cnt) {
        const int t = pair_list[p0 + n] / k;
        v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H + g * kGK + c * 8));
      }
      uint4 o;  // K order (0,4,1,5,2,6,3,7)
      o.x = prmt(v.x, v.z, 0x5410u);
      o.y = prmt(v.x, v.z, 0x7632u);
      o.z = prmt(v.y, v.w, 0x5410u);
      o.w = prmt(v.y, v.w, 0x7632u);
      const int pos = base + n;
      *reinterpret_cast<uint4*>(xp + ((size_t)g * pcap + pos) * kGK + ((c ^ (pos & 7)) * 8)) = o;
    }
  }
}

// ------------------------------------------------------------------ GEMMs ---
struct GroupedArgs {
  const uint16_t* bp;    // packed activations [K/64][pcap][64] (x or h)
  const int* unique;     // [u] distinct experts, ascending
  const int* offsets;    // [u + 1]
  const int* padded;     // [u + 1] padded row offsets of the packed layout
  const int* num_unique; // [1]
  const uint32_t* q[2];  // codes of matrix 0 / 1 of a tile
  const uint16_t* s[2];  // scales
  const uint16_t* b[2];  // biases
  int roff[2];           // row offset of matrix m inside the tile (0/0 or 0/128)
  uint16_t* hp;          // phase 0: packed h [I/64][pcap][64]
  float* y;              // phase 1: [P, H] fp32 in pair_list order
  int rows, K, mrows;    // weight rows per expert; K; weight rows per tile
  int pcap, H;
};

// Shared-memory matrix descriptor for the A tile of matrix m in A buffer ab.
__device__ __forceinline__ uint32_t a_tile(const unsigned char* base, uint32_t ab, int m) {
  return smem_u32(base + ab * kGABytes + m * kGATile);
}

template <int PHASE, int NMAX>
__global__ void __launch_bounds__(kGThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GroupedArgs a) {
  using C = GCfg<NMAX>;
  extern __shared__ __align__(128) unsigned char gsm_raw[];
  __shared__ __align__(8) uint64_t full[C::kStages], w_empty[C::kStages];
  __shared__ __align__(8) uint64_t a_full[kGABufs], a_empty[kGABufs];
  __shared__ __align__(8) uint64_t acc_full[kGAccBufs], acc_empty[kGAccBufs];
  __shared__ uint32_t tmem_base_s;
  // swizzled tiles start at 1024-byte boundaries of the shared address space
  unsigned char* gsm = gsm_raw + ((1024u - (smem_u32(gsm_raw) & 1023u)) & 1023u);
  unsigned char* abuf = gsm;                                // A buffers
  unsigned char* ring = gsm + kGABufs * kGABytes;           // copy stages
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1 + 32);         // expect_tx + one cp.async arrival per lane
      mbar_init(&w_empty[i], kGDeq + 1);   // dequantising warps + the MMA commit
    }
    for (int i = 0; i < kGABufs; ++i) {
      mbar_init(&a_full[i], kGDeq);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < kGAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kGEpi);
    }
    fence_barrier_init();
  }
  if (warp == kGMmaWarp) {
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
  uint32_t tc = 0;  // chunk tiles started

  if (warp == kGProducer) {
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
            if (round > 0) ok = mbar_wait(&w_empty[st], (round - 1) & 1);
            if (ok) mbar_arrive_expect_tx(&full[st], kGSlabsPerStage * np * (kGK * 2));
          }
          ok = __shfl_sync(kFull, ok, 0);
          if (!ok) break;
          unsigned char* stg = ring + st * C::kStageBytes;
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
            cp_async4(stg + C::kOffS + rr * 4, a.s[m] + row * (a.K / kGK) + j0);
            cp_async4(stg + C::kOffBias + rr * 4, a.b[m] + row * (a.K / kGK) + j0);
          }
          if (lane == 0) {
#pragma unroll
            for (int jj = 0; jj < kGSlabsPerStage; ++jj) {
              const size_t prow = (size_t)(j0 + jj) * a.pcap + pp0 + c0;
              bulk_g2s(stg + C::kOffB + jj * C::kBTile, a.bp + prow * kGK, np * kGK * 2,
                       &full[st]);
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
  } else if (warp == kGMmaWarp) {
    // ---------------------------------------------------------- MMA issuer ---
    // The whole warp runs this loop (operands warp-uniform); one elected lane issues.
    bool issued_any = false;
    uint32_t last_db = 0, last_tc = 0;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int slot = tile / mtiles;
      const int cnt = a.offsets[slot + 1] - a.offsets[slot];
      for (int c0 = 0; c0 < cnt && ok; c0 += C::kN, ++tc) {
        const int np = (min(C::kN, cnt - c0) + 15) & ~15;
        const uint32_t idesc = f16_idesc(kGM, np);
        const uint32_t db = tc % kGAccBufs;
        if (tc >= (uint32_t)kGAccBufs)
          ok = __all_sync(kFull, mbar_wait(&acc_empty[db], (tc / kGAccBufs - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        bool first = true;
        for (int j0 = 0; j0 < nslab && ok; j0 += kGSlabsPerStage, ++sc) {
          const int st = sc % C::kStages;
          ok = __all_sync(kFull, mbar_wait(&full[st], (sc / C::kStages) & 1));
          const uint32_t bbase = smem_u32(ring + st * C::kStageBytes + C::kOffB);
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
                tc_mma_ss_elect(tmem + C::col_d(db, m), sw128_desc(a_tile(abuf, ab, m) + kk * 32),
                                bdesc, idesc, (first && kk == 0) ? 0u : 1u);
            }
            first = false;
            tc_commit_elect(&a_empty[ab]);
            if (jj == kGSlabsPerStage - 1) tc_commit_elect(&w_empty[st]);
          }
        }
        if (!ok) break;
        tc_commit_elect(&acc_full[db]);
        issued_any = true;
        last_db = db;
        last_tc = tc;
      }
    }
    // no MMA may run past the deallocation below (at once when all went well)
    if (issued_any) mbar_wait(&acc_full[last_db], (last_tc / kGAccBufs) & 1);
  } else if (warp < kGDeq) {
    // ----------------------------------------------------------- dequantise ---
    const int m = warp >> 2, r = 32 * (warp & 3) + lane;
    const uint32_t one2 = 0x3F803F80u, m128 = 0xC300C300u;  // bf16 pairs (1, 1), (-128, -128)
    const unsigned arow = (unsigned)((r >> 3) * 1024 + (r & 7) * 128);
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int slot = tile / mtiles;
      const int cnt = a.offsets[slot + 1] - a.offsets[slot];
      for (int c0 = 0; c0 < cnt && ok; c0 += C::kN) {
        for (int j0 = 0; j0 < nslab && ok; j0 += kGSlabsPerStage, ++sc) {
          const int st = sc % C::kStages;
          ok = __all_sync(kFull, mbar_wait(&full[st], (sc / C::kStages) & 1));
          if (!ok) break;
          const unsigned char* stg = ring + st * C::kStageBytes;
          const uint4* crow = reinterpret_cast<const uint4*>(stg + (m * kGM + r) * kGCodePitch);
          const uint32_t sv2 = *reinterpret_cast<const uint32_t*>(stg + C::kOffS + (m * kGM + r) * 4);
          const uint32_t bv2 =
              *reinterpret_cast<const uint32_t*>(stg + C::kOffBias + (m * kGM + r) * 4);
          for (int jj = 0; jj < kGSlabsPerStage && ok; ++jj, ++gs) {
            const uint32_t ab = gs % kGABufs;
            if (gs >= (uint32_t)kGABufs)
              ok = __all_sync(kFull, mbar_wait(&a_empty[ab], (gs / kGABufs - 1) & 1));
            if (!ok) break;
            // this slab's scale and bias in both halves of a bf16 pair
            const uint32_t s2 = jj ? __byte_perm(sv2, 0, 0x3232) : __byte_perm(sv2, 0, 0x1010);
            const uint32_t b2 = jj ? __byte_perm(bv2, 0, 0x3232) : __byte_perm(bv2, 0, 0x1010);
            const uint4 w0 = crow[2 * jj], w1 = crow[2 * jj + 1];
            unsigned char* dst = abuf + ab * kGABytes + m * kGATile + arow;
            const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(dst + ((c ^ (r & 7)) << 4)) =
                  dequant_word(wv[c], one2, m128, s2, b2);
            fence_proxy_async();  // the generic-proxy stores, before the MMA reads them
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[ab]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&w_empty[st]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue ---
    const int qd = warp - kGDeq, r = 32 * qd + lane;  // tensor-memory lane quarter qd
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int slot = tile / mtiles, m0 = (tile % mtiles) * a.mrows;
      const int p0 = a.offsets[slot], cnt = a.offsets[slot + 1] - p0;
      const int pp0 = a.padded[slot];
      for (int c0 = 0; c0 < cnt && ok; c0 += C::kN, ++tc) {
        const int n = min(C::kN, cnt - c0), np = (n + 15) & ~15;
        const uint32_t db = tc % kGAccBufs;
        ok = __all_sync(kFull, mbar_wait(&acc_full[db], (tc / kGAccBufs) & 1));
        if (!ok) break;
        tc_fence_after();
        if (PHASE == 0) {
          // h = bf16(silu(bf16 g) * bf16 u): matrix 0 holds g, matrix 1 u; this
          // thread's row of the tile is column m0 + r of h
          const int irow = m0 + r;
          const int gI = irow / kGK, ci = irow % kGK;
          const int pin = (ci & ~7) + 2 * (ci & 3) + ((ci >> 2) & 1);  // K order position
#pragma unroll 1
          for (int c16 = 0; c16 < np; c16 += 16) {
            uint32_t gr[16], ur[16];
            tc_ld16(tmem + C::col_d(db, 0) + c16 + lane_base, gr);
            tc_ld16(tmem + C::col_d(db, 1) + c16 + lane_base, ur);
            tc_wait_ld();
            tc_regs_ready(gr);
            tc_regs_ready(ur);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g = round_to_bf16(__uint_as_float(gr[i]));
              const float uu = round_to_bf16(__uint_as_float(ur[i]));
              const uint16_t hb = float_to_bf16_bits(g / (1.0f + __expf(-g)) * uu);
              const int pos = pp0 + c0 + c16 + i;
              a.hp[((size_t)gI * a.pcap + pos) * kGK + (((pin >> 3) ^ (pos & 7)) << 3) +
                   (pin & 7)] = hb;
            }
          }
        } else {
          // y rows of the chunk's pairs (pair_list order), fp32: rows m0 + r and
          // m0 + 128 + r of the expert's Wd
#pragma unroll 1
          for (int mm = 0; mm < 2; ++mm) {
            float* yo = a.y + (size_t)(p0 + c0) * a.H + m0 + a.roff[mm] + r;
#pragma unroll 1
            for (int c16 = 0; c16 < np; c16 += 16) {
              uint32_t yr[16];
              tc_ld16(tmem + C::col_d(db, mm) + c16 + lane_base, yr);
              tc_wait_ld();
              tc_regs_ready(yr);
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (c16 + i < n) yo[(size_t)(c16 + i) * a.H] = __uint_as_float(yr[i]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[db]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kGMmaWarp) {
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
