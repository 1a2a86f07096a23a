// Device helpers shared by the kernels: mbarriers, 1-D bulk copies, grid
// dependency control, bounded waits, bf16 bit helpers and the error word.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace qeg {

constexpr unsigned kFull = 0xffffffffu;

// Error bits the kernels set instead of trapping (read by moe_read_device_status).
constexpr unsigned kErrExpertIndex = 1u;
constexpr unsigned kErrTimeout = 2u;

// One word per device; set with atomicOr, read and cleared by the host.
__device__ unsigned int g_error_word;

__device__ __forceinline__ void set_error(unsigned bits) { atomicOr(&g_error_word, bits); }

// Limit for every spin on an mbarrier or a counter: far beyond any legitimate wait.
// g_wait_limit_ns is the limit in force (moe_set_wait_limit_ns may shorten it, so that
// a test can make a wait run out); kWaitLimitNs stays the bound of the waits that let
// copies and MMAs already in flight finish before a CTA exits.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;

__device__ __forceinline__ unsigned long long wait_limit() {
  return *static_cast<volatile unsigned long long*>(&g_wait_limit_ns);
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Test phase `parity` of `bar`; a thread whose phase is not complete is suspended
// until it completes or about kSuspendNs pass, instead of spinning on issue slots.
constexpr unsigned kSuspendNs = 1000000;  // 1 ms
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most `limit` ns (the limit in
// force by default).  Returns false (and sets kErrTimeout) if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity,
                                          unsigned long long limit = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  if (limit == 0) limit = wait_limit();
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit) {
      set_error(kErrTimeout);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> shared, completing `bytes` of transaction count on
// `bar`.  dst, src and bytes must be multiples of 16.  Local memory only, no
// cluster multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// The same for data read once (a weight stream): the lines are marked evict-first in
// L2, so the stream does not push out what is read again (the kernel's code, its
// tables, h and y).  On B200 this shortened the small-window layer by about 3 %.
__device__ __forceinline__ void bulk_g2s_stream(void* dst, const void* src, unsigned bytes,
                                                uint64_t* bar) {
  asm volatile(
      "{\n .reg .b64 pol;\n createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n"
      " cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], pol;\n}" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Programmatic dependent launch controls.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses (and those the
// preceding barrier made visible) before its following async-proxy copies.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_barrier(unsigned id, unsigned threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Arrive at a named barrier without waiting (the waiting side uses named_barrier).
__device__ __forceinline__ void named_barrier_arrive(unsigned id, unsigned threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ float bf16_bits_to_float(uint16_t v) {
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

// fp32 -> bf16 bits, round to nearest even (NaN kept quiet).
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return static_cast<uint16_t>((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

__device__ __forceinline__ float round_to_bf16(float f) {
  return bf16_bits_to_float(float_to_bf16_bits(f));
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Warp reduce-scatter of V values (V a power of two, <= 32): afterwards the
// lanes whose low (5 - log2 V) bits are zero each hold the full warp sum of one
// value, whose index is returned.  Sums run in a fixed order (deterministic).
template <int V>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[V], int lane, int& vid) {
  vid = 0;
#pragma unroll
  for (int width = V, mask = 16; width > 1; width >>= 1, mask >>= 1) {
    const bool upper = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < width / 2; ++i) {
      const float keep = upper ? v[i + width / 2] : v[i];
      const float send = upper ? v[i] : v[i + width / 2];
      v[i] = keep + __shfl_xor_sync(kFull, send, mask);
    }
    if (upper) vid += width / 2;
  }
  constexpr int kSteps = (V >= 32) ? 0 : (V >= 16 ? 1 : (V >= 8 ? 2 : (V >= 4 ? 3 : (V >= 2 ? 4 : 5))));
#pragma unroll
  for (int s = 0; s < kSteps; ++s) v[0] += __shfl_xor_sync(kFull, v[0], 1 << (kSteps - 1 - s));
  return v[0];
}

}  // namespace qeg
