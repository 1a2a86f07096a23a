// Seeded synthetic expert banks, device side.
//
// The same generator as synth_host.c (SplitMix64 counter stream, the
// sum-of-twelve-uniforms normal draw, the min/max affine group-64 quantiser and
// the LSB-first nibble packing), written with explicitly rounded IEEE
// operations (__fsub_rn, __fdiv_rn, __fmul_rn) and no contraction, so a bank
// filled here holds the same bits as one drawn on the host.  It exists so that
// multi-gigabyte banks can be drawn in milliseconds; it holds none of the
// layer's arithmetic.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t sm64_at(uint64_t seed, uint64_t n) {
  return mix64(seed + (n + 1) * kGamma);
}

__device__ __forceinline__ float normal_draw(uint64_t key, uint64_t elem) {
  uint32_t acc = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    uint64_t r = sm64_at(key, 3 * elem + (uint64_t)i);
    acc += (uint32_t)(r & 0xFFFF) + (uint32_t)((r >> 16) & 0xFFFF) +
           (uint32_t)((r >> 32) & 0xFFFF) + (uint32_t)(r >> 48);
  }
  return __fsub_rn(__fmul_rn(__uint2float_rn(acc), 1.0f / 65536.0f), 6.0f);
}

__device__ __forceinline__ uint16_t bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float((uint32_t)b << 16);
}

// One thread per (expert-list entry, row, group of 64 columns).
__global__ void fill_bank_kernel(uint32_t* __restrict__ q, uint16_t* __restrict__ s,
                                 uint16_t* __restrict__ b, int rows, int cols, uint64_t key,
                                 const int32_t* __restrict__ experts, int n_experts) {
  const int gpr = cols / 64;
  const uint64_t per_expert = (uint64_t)rows * gpr;
  const uint64_t total = per_expert * (uint64_t)n_experts;
  for (uint64_t gid = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; gid < total;
       gid += (uint64_t)gridDim.x * blockDim.x) {
    const int ei = (int)(gid / per_expert);
    const uint64_t rem = gid % per_expert;
    const int r = (int)(rem / gpr), g = (int)(rem % gpr);
    const int e = experts ? experts[ei] : ei;
    const uint64_t elem0 = ((uint64_t)e * rows + r) * cols + (uint64_t)g * 64;
    float mn = 0.f, mx = 0.f;
    for (int c = 0; c < 64; ++c) {
      float w = normal_draw(key, elem0 + c);
      if (c == 0 || w < mn) mn = w;
      if (c == 0 || w > mx) mx = w;
    }
    uint16_t sb = (mx == mn) ? (uint16_t)0x3F80 : bf16_rne(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
    if ((sb & 0x7FFF) == 0) sb = 0x3F80;
    const uint16_t bb = bf16_rne(mn);
    const float sf = bf16_to_f32(sb), bf = bf16_to_f32(bb);
    uint32_t* qrow = q + ((uint64_t)e * rows + r) * (cols / 8) + (uint64_t)g * 8;
    for (int wd = 0; wd < 8; ++wd) {
      uint32_t word = 0;
      for (int j = 0; j < 8; ++j) {
        // Draw again rather than keep 64 floats live: the draw is a pure function.
        const float w = normal_draw(key, elem0 + wd * 8 + j);
        int qi = (mx == mn) ? 0 : (int)rintf(__fdiv_rn(__fsub_rn(w, bf), sf));
        qi = qi < 0 ? 0 : (qi > 15 ? 15 : qi);
        word |= (uint32_t)qi << (4 * j);
      }
      qrow[wd] = word;
    }
    s[((uint64_t)e * rows + r) * gpr + g] = sb;
    b[((uint64_t)e * rows + r) * gpr + g] = bb;
  }
}

// mxfp4 encoding, the device twin of synth_group_mx in synth_host.c (e8m0 scale
// per 32 columns from the group's largest magnitude, e2m1 codes nearest, ties to
// the even mantissa, saturating at 6).
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  const float a = fabsf(v);
  uint32_t m;
  if (a <= 0.25f) m = 0;
  else if (a < 0.75f) m = 1;
  else if (a <= 1.25f) m = 2;
  else if (a < 1.75f) m = 3;
  else if (a <= 2.5f) m = 4;
  else if (a < 3.5f) m = 5;
  else if (a <= 5.0f) m = 6;
  else m = 7;
  return (v < 0.0f ? 8u : 0u) | m;
}

__global__ void fill_bank_mx_kernel(uint32_t* __restrict__ q, uint8_t* __restrict__ e8,
                                    int rows, int cols, uint64_t key,
                                    const int32_t* __restrict__ experts, int n_experts) {
  const int gpr = cols / 32;
  const uint64_t per_expert = (uint64_t)rows * gpr;
  const uint64_t total = per_expert * (uint64_t)n_experts;
  for (uint64_t gid = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; gid < total;
       gid += (uint64_t)gridDim.x * blockDim.x) {
    const int ei = (int)(gid / per_expert);
    const uint64_t rem = gid % per_expert;
    const int r = (int)(rem / gpr), g = (int)(rem % gpr);
    const int e = experts ? experts[ei] : ei;
    const uint64_t elem0 = ((uint64_t)e * rows + r) * cols + (uint64_t)g * 32;
    float amax = 0.f;
    for (int c = 0; c < 32; ++c) amax = fmaxf(amax, fabsf(normal_draw(key, elem0 + c)));
    const int ex = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127 - 2 : 0;
    const float inv = __uint_as_float((uint32_t)(127 - ex) << 23);
    uint32_t* qrow = q + ((uint64_t)e * rows + r) * (cols / 8) + (uint64_t)g * 4;
    for (int wd = 0; wd < 4; ++wd) {
      uint32_t word = 0;
      for (int j = 0; j < 8; ++j) {
        const float w = normal_draw(key, elem0 + wd * 8 + j);
        word |= (amax > 0.f ? e2m1_code(__fmul_rn(w, inv)) : 0u) << (4 * j);
      }
      qrow[wd] = word;
    }
    e8[((uint64_t)e * rows + r) * gpr + g] = (uint8_t)(127 + ex);
  }
}

}  // namespace

// Host-side copy of the stream key derivation (plain integer arithmetic).
static uint64_t host_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

extern "C" {

// Fill experts `experts[0..n_experts)` (device int32 list; null = experts
// 0..n_experts-1) of a device bank q [E, rows, cols/8], s/b [E, rows, cols/64],
// drawn from stream (seed, matrix_id), asynchronously on `stream`.
// Returns 0, -1 on bad arguments, or the CUDA error code of the launch.
int synth_dev_fill_bank(uint32_t* q, uint16_t* s, uint16_t* b, int rows, int cols, uint64_t seed,
                        uint64_t matrix_id, const int32_t* experts, int n_experts, void* stream) {
  if (!q || !s || !b || rows <= 0 || cols <= 0 || cols % 64 || n_experts <= 0) return -1;
  const uint64_t key = host_mix64(seed + (matrix_id + 1) * 0x9E3779B97F4A7C15ULL);
  const uint64_t total = (uint64_t)rows * (cols / 64) * (uint64_t)n_experts;
  const int threads = 256;
  uint64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148ull * 64) blocks = 148ull * 64;
  fill_bank_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
      q, s, b, rows, cols, key, experts, n_experts);
  return (int)cudaGetLastError();
}

// The mxfp4 twin of synth_dev_fill_bank: q [E, rows, cols/8] e2m1 codes and
// e8 [E, rows, cols/32] e8m0 scales (cols a multiple of 32), bit-identical to
// synth_fill_bank_mxfp4 on the host.
int synth_dev_fill_bank_mxfp4(uint32_t* q, uint8_t* e8, int rows, int cols, uint64_t seed,
                              uint64_t matrix_id, const int32_t* experts, int n_experts,
                              void* stream) {
  if (!q || !e8 || rows <= 0 || cols <= 0 || cols % 32 || n_experts <= 0) return -1;
  const uint64_t key = host_mix64(seed + (matrix_id + 1) * 0x9E3779B97F4A7C15ULL);
  const uint64_t total = (uint64_t)rows * (cols / 32) * (uint64_t)n_experts;
  const int threads = 256;
  uint64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148ull * 64) blocks = 148ull * 64;
  fill_bank_mx_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
      q, e8, rows, cols, key, experts, n_experts);
  return (int)cudaGetLastError();
}

}  // extern "C"
