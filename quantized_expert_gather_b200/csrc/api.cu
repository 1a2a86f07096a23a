// C ABI of the union-of-experts quantized SwitchGLU library (include/moe_qeg.h):
// argument validation, workspace layout, path selection and kernel launches.
// Everything here is host code; the arithmetic is in the kernels.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/moe_qeg.h"
#include "common.cuh"
#include "layer.cuh"
#include "route_union.cuh"
#include "grouped.cuh"
#include "router.cuh"

namespace qeg {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kNumKernels = 22;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int smem_optin = 0;
  // dynamic shared memory limit: layer (affine), route_union, grouped gate+up and down
  // (chunks of 64 pairs), combine, grouped gate+up and down (chunks of 96, then of 32
  // pairs), layer (mxfp4); then the layer instances for fixed widths (affine 4096/2048,
  // mxfp4 6144/2048 and 4096/2048, each also with resident x rows), which share the
  // general instances' limits; then the grouped kernels for mxfp4 banks (chunks of 64,
  // 96, 32 pairs), which share the affine ones'
  int dyn_smem[kNumKernels] = {};
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
thread_local const char* g_last_error = "no error";

moe_status cuda_fail(cudaError_t e) {
  g_last_error = cudaGetErrorString(e);
  return MOE_ERR_CUDA;
}

// Per-device state: SM count, shared-memory limit, kernel attributes set once.
moe_status device_info(DeviceInfo** out) {
  int dev = 0;
  const cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return cuda_fail(ge);
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    cudaError_t e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    // dynamic + static shared memory may not exceed the opt-in limit
    const void* kernels[kNumKernels] = {
                              reinterpret_cast<const void*>(layer_kernel<kFmtAffine>),
                              reinterpret_cast<const void*>(route_union_kernel),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<0, 64>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<1, 64>),
                              reinterpret_cast<const void*>(grouped_combine_kernel),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<0, 96>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<1, 96>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<0, 32>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<1, 32>),
                              reinterpret_cast<const void*>(layer_kernel<kFmtMx>),
                              reinterpret_cast<const void*>(layer_kernel<kFmtAffine, 4, 2>),
                              reinterpret_cast<const void*>(layer_kernel<kFmtMx, 6, 2>),
                              reinterpret_cast<const void*>(layer_kernel<kFmtMx, 4, 2>),
                              reinterpret_cast<const void*>(layer_kernel<kFmtAffine, 4, 2, 1>),
                              reinterpret_cast<const void*>(layer_kernel<kFmtMx, 6, 2, 1>),
                              reinterpret_cast<const void*>(layer_kernel<kFmtMx, 4, 2, 1>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<0, 64, kFmtMx>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<1, 64, kFmtMx>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<0, 96, kFmtMx>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<1, 96, kFmtMx>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<0, 32, kFmtMx>),
                              reinterpret_cast<const void*>(grouped_gemm_kernel<1, 32, kFmtMx>)};
    for (int i = 0; i < kNumKernels; ++i) {
      cudaFuncAttributes fa;
      cudaError_t e = cudaFuncGetAttributes(&fa, kernels[i]);
      if (e == cudaSuccess) {
        d.dyn_smem[i] = d.smem_optin - static_cast<int>(fa.sharedSizeBytes);
        e = cudaFuncSetAttribute(kernels[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 d.dyn_smem[i]);
      }
      if (e != cudaSuccess) return cuda_fail(e);
    }
    d.ready = true;
  }
  *out = &d;
  return MOE_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool shape_ok(int T, int k, int E, int hidden, int inter) {
  if (T <= 0 || k <= 0 || E <= 0 || hidden <= 0 || inter <= 0) return false;
  if (hidden % 64 || inter % 64) return false;
  if ((long long)T * k > MOE_MAX_PAIRS) return false;
  return true;
}

bool shape_supported(int T, int k, int E, int hidden, int inter) {
  return E <= MOE_MAX_EXPERTS && hidden <= MOE_MAX_DIM && inter <= MOE_MAX_DIM;
}

struct WsLayout {
  size_t barrier, num_unique, unique, offsets, pair_list, h, y;  // barrier = counters
  size_t padded, xs, hs, xp, hp, pcap;   // grouped path: packed activations and sums
  size_t total;
};

// 1 = the persistent fused kernel (small windows), 2 = the grouped tensor-core
// kernels (windows with more pairs; hidden a multiple of 256, inter of 128),
// 0 = neither.  Both bank formats take both paths.
// `routed`: the router step runs inside the persistent kernel (its picks and weights
// take shared memory too).
int select_path(int T, int k, int E, int hidden, int inter, int fmt = kFmtAffine,
                bool routed = false) {
  if (!shape_ok(T, k, E, hidden, inter) || !shape_supported(T, k, E, hidden, inter)) return 0;
  if (T * k <= kMaxPairsFused) {
    LayerGeom g = layer_geom(hidden, inter, fmt);
    if (layer_plan(g, E, T, k, kSmemBudget, routed)) return 1;
  }
  // the grouped path: hidden a multiple of 256 (down tiles), inter a multiple of 128
  // (gate/up tiles)
  if (hidden % (2 * kGM) == 0 && inter % (2 * kGK) == 0 &&
      route_union_smem_bytes(E) <= kSmemBudget && sizeof(int) * (size_t)T * k <= kSmemBudget)
    return 2;
  return 0;
}

WsLayout ws_layout(int T, int k, int E, int hidden, int inter, int fmt = kFmtAffine) {
  const size_t P = (size_t)T * k;
  const size_t m = P < (size_t)E ? P : (size_t)E;
  WsLayout w;
  w.barrier = 0;
  w.num_unique = align_up(4 * kSyncWords, 256);
  w.unique = w.num_unique + 16;
  w.offsets = align_up(w.unique + 4 * m, 16);
  w.pair_list = align_up(w.offsets + 4 * (m + 1), 16);
  w.h = align_up(w.pair_list + 4 * P, 256);
  w.y = align_up(w.h + 2 * P * (size_t)inter, 256);
  const size_t tail = align_up(w.y + 4 * P * (size_t)hidden, 256);
  const size_t total1 = tail;  // the persistent kernel needs nothing more
  // grouped path: every expert's pairs padded to 16 rows
  w.pcap = align_up(P + 15 * m, 16);
  w.padded = tail;
  w.xs = align_up(w.padded + 4 * (m + 1), 256);
  w.hs = align_up(w.xs + 4 * (size_t)(hidden / kGK) * w.pcap, 256);
  w.xp = align_up(w.hs + 4 * (size_t)(inter / kGK) * w.pcap, 256);
  w.hp = align_up(w.xp + 2 * (size_t)hidden * w.pcap, 256);
  const size_t total2 = align_up(w.hp + 2 * (size_t)inter * w.pcap, 256);
  w.total = select_path(T, k, E, hidden, inter, fmt) == 2 ? total2 : total1;
  return w;
}

template <int F>
cudaError_t launch_layer(const uint16_t* x, const int32_t* idx, const float* w,
                         const uint32_t* gq, const uint16_t* gs, const uint16_t* gb,
                         const uint32_t* uq, const uint16_t* us, const uint16_t* ub,
                         const uint32_t* dq, const uint16_t* ds, const uint16_t* db, int T, int k,
                         int E, int H, int I, uint16_t* out, unsigned char* ws,
                         const DeviceInfo& d, cudaStream_t st, moe_status* why,
                         const float* logits = nullptr, int renorm = 0,
                         int32_t* ridx_out = nullptr, float* rw_out = nullptr) {
  const WsLayout wl = ws_layout(T, k, E, H, I);
  LayerArgs a;
  a.logits = logits;  // the fused router step (idx and w unused then)
  a.renorm = renorm;
  a.ridx_out = ridx_out;
  a.rw_out = rw_out;
  a.x = x;
  a.idx = idx;
  a.w = w;
  a.gq = gq;
  a.gs = gs;
  a.gb = gb;
  a.uq = uq;
  a.us = us;
  a.ub = ub;
  a.dq = dq;
  a.ds = ds;
  a.db = db;
  a.h = reinterpret_cast<uint16_t*>(ws + wl.h);
  a.y = reinterpret_cast<float*>(ws + wl.y);
  a.sync = reinterpret_cast<unsigned*>(ws + wl.barrier);
  a.ex_u = reinterpret_cast<int*>(ws + wl.num_unique);
  a.ex_unique = reinterpret_cast<int*>(ws + wl.unique);
  a.ex_offsets = reinterpret_cast<int*>(ws + wl.offsets);
  a.ex_pair_list = reinterpret_cast<int*>(ws + wl.pair_list);
  a.out = out;
  a.T = T;
  a.k = k;
  a.E = E;
  a.H = H;
  a.I = I;
  a.g = layer_geom(H, I, F);
  a.wait_prior = 1;
  const int ki = F == kFmtMx ? 9 : 0;  // dyn_smem index of this layer kernel
  if (!layer_plan(a.g, E, T, k, (size_t)d.dyn_smem[ki], logits != nullptr)) {
    *why = MOE_ERR_UNSUPPORTED;
    return cudaSuccess;
  }
  // the fused router stages one logit row per routing warp behind the tables
  if (logits && (size_t)kRouteWarps * ((5u * (unsigned)E + 15u) & ~15u) > a.g.total - a.g.tables) {
    *why = MOE_ERR_UNSUPPORTED;
    return cudaSuccess;
  }
  // the window's x rows fit the normal activation area: each CTA keeps them all
  a.x_res = (size_t)T * act_bytes(a.g.rounds_a) <= a.g.act_n ? 1 : 0;
  // One CTA per SM, all resident at once (the kernel has grid barriers); the
  // launch may overlap the tail of the preceding kernel (programmatic launch).
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(d.sms);
  c.blockDim = dim3(kThreads);
  c.dynamicSmemBytes = a.g.total;
  c.stream = st;
  c.attrs = attr;
  c.numAttrs = 2;
  // the instance with the chunk rounds fixed, for the widths that have one
  // (and x resident: the instance without phase-A activation sets)
  const int ra = a.g.rounds_a, rb = a.g.rounds_b;
  if (ra == 4 && rb == 2)
    return a.x_res ? cudaLaunchKernelEx(&c, layer_kernel<F, 4, 2, 1>, a)
                   : cudaLaunchKernelEx(&c, layer_kernel<F, 4, 2>, a);
  if constexpr (F == kFmtMx) {
    if (ra == 6 && rb == 2)
      return a.x_res ? cudaLaunchKernelEx(&c, layer_kernel<F, 6, 2, 1>, a)
                     : cudaLaunchKernelEx(&c, layer_kernel<F, 6, 2>, a);
  }
  return cudaLaunchKernelEx(&c, layer_kernel<F>, a);
}

// The grouped path: route-union (with padded offsets), x packing, gate+up, down
// and combine as five launches on `st` (no host synchronisation).  The union
// arrays, the packed activations, their sums and y live in the workspace.
template <int F>
cudaError_t launch_grouped(const uint16_t* x, const int32_t* idx, const float* w,
                           const uint32_t* gq, const uint16_t* gs, const uint16_t* gb,
                           const uint32_t* uq, const uint16_t* us, const uint16_t* ub,
                           const uint32_t* dq, const uint16_t* ds, const uint16_t* db, int T,
                           int k, int E, int H, int I, uint16_t* out, unsigned char* ws,
                           const DeviceInfo& d, cudaStream_t st, moe_status* why) {
  const WsLayout wl = ws_layout(T, k, E, H, I, F);
  const int P = T * k;
  int* nu = reinterpret_cast<int*>(ws + wl.num_unique);
  int* uniq = reinterpret_cast<int*>(ws + wl.unique);
  int* offs = reinterpret_cast<int*>(ws + wl.offsets);
  int* plist = reinterpret_cast<int*>(ws + wl.pair_list);
  float* y = reinterpret_cast<float*>(ws + wl.y);
  int* padded = reinterpret_cast<int*>(ws + wl.padded);
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + wl.xp);
  uint16_t* hp = reinterpret_cast<uint16_t*>(ws + wl.hp);
  float* xs = reinterpret_cast<float*>(ws + wl.xs);
  float* hs = reinterpret_cast<float*>(ws + wl.hs);
  const int pcap = static_cast<int>(wl.pcap);
  const int m = P < E ? P : E;
  const size_t usmem = route_union_smem_bytes(E);
  const size_t csmem = sizeof(int) * (size_t)P;
  // pairs per MMA chunk: 96 when experts average more than 40 pairs (fewer weight
  // re-reads), 32 when they average at most 20 (more accumulator buffers), else 64
  const int width = P > 40 * m ? 96 : (P <= 20 * m ? 32 : 64);
  const unsigned gsmem = width == 96 ? GCfg<96>::kSmem : width == 32 ? GCfg<32>::kSmem : GCfg<64>::kSmem;
  // dyn_smem index of the gate+up kernel (down: the next one)
  const int ki = F == kFmtMx ? (width == 96 ? 18 : width == 32 ? 20 : 16)
                             : (width == 96 ? 5 : width == 32 ? 7 : 2);
  const int grid = width == 32 ? 2 * d.sms : d.sms;
  if (usmem > (size_t)d.dyn_smem[1] || csmem > (size_t)d.dyn_smem[4] ||
      gsmem > (unsigned)d.dyn_smem[ki] || gsmem > (unsigned)d.dyn_smem[ki + 1]) {
    *why = MOE_ERR_UNSUPPORTED;
    return cudaSuccess;
  }
  route_union_kernel<<<1, 32 * kUnionWarps, usmem, st>>>(idx, P, E, uniq, offs, plist, nu,
                                                         padded);
  // blocks (slot, slice): up to two per SM along the slots, four slices of each slot
  const dim3 pgrid(m < 2 * d.sms ? m : 2 * d.sms, 4);
  grouped_pack_x_kernel<<<pgrid, 256, 0, st>>>(x, plist, offs, padded, nu, k, H, pcap, xp, xs);
  GroupedArgs g{};
  g.unique = uniq;
  g.offsets = offs;
  g.padded = padded;
  g.num_unique = nu;
  g.pcap = pcap;
  g.H = H;
  g.hp = hp;
  g.hs = hs;
  g.y = y;
  // gate + up: 128 rows of Wg and the same 128 rows of Wu per tile, K = H, packed x
  g.bp = xp;
  g.bs = xs;
  g.q[0] = gq;
  g.s[0] = gs;
  g.b[0] = gb;
  g.q[1] = uq;
  g.s[1] = us;
  g.b[1] = ub;
  g.roff[0] = g.roff[1] = 0;
  g.rows = I;
  g.K = H;
  g.mrows = kGM;
  if (width == 96)
    grouped_gemm_kernel<0, 96, F><<<grid, kGThreads, gsmem, st>>>(g);
  else if (width == 32)
    grouped_gemm_kernel<0, 32, F><<<grid, kGThreads, gsmem, st>>>(g);
  else
    grouped_gemm_kernel<0, 64, F><<<grid, kGThreads, gsmem, st>>>(g);
  // down: 256 rows of Wd per tile (two 128-row matrices), K = I, packed h
  g.bp = hp;
  g.bs = hs;
  g.q[0] = g.q[1] = dq;
  g.s[0] = g.s[1] = ds;
  g.b[0] = g.b[1] = db;
  g.roff[1] = kGM;
  g.rows = H;
  g.K = I;
  g.mrows = 2 * kGM;
  if (width == 96)
    grouped_gemm_kernel<1, 96, F><<<grid, kGThreads, gsmem, st>>>(g);
  else if (width == 32)
    grouped_gemm_kernel<1, 32, F><<<grid, kGThreads, gsmem, st>>>(g);
  else
    grouped_gemm_kernel<1, 64, F><<<grid, kGThreads, gsmem, st>>>(g);
  grouped_combine_kernel<<<2 * d.sms, kGCombineThreads, csmem, st>>>(y, w, plist, offs, nu, T, k,
                                                                      H, out);
  return cudaGetLastError();
}

struct OwnedWorkspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
OwnedWorkspace g_ws[kMaxDevices];

// The library-owned workspace of the current device, grown (outside stream
// capture only) to hold this shape; zeroed when allocated.
moe_status owned_workspace(int T, int k, int E, int hidden, int inter, int fmt, void* stream,
                           void** out, size_t* bytes) {
  int dev = 0;
  const cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return cuda_fail(ge);
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  const size_t need = ws_layout(T, k, E, hidden, inter, fmt).total;
  OwnedWorkspace& w = g_ws[dev];
  std::lock_guard<std::mutex> lock(g_mu);
  if (w.bytes < need) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const cudaError_t ce = cudaStreamIsCapturing((cudaStream_t)stream, &cs);
    if (ce != cudaSuccess) return cuda_fail(ce);
    if (cs != cudaStreamCaptureStatusNone) return MOE_ERR_WORKSPACE;
    // The old buffer may still be in use by queued work on some stream.
    if (w.ptr) {
      const cudaError_t se = cudaDeviceSynchronize();
      if (se != cudaSuccess) return cuda_fail(se);
      cudaFree(w.ptr);
      w.ptr = nullptr;
      w.bytes = 0;
    }
    cudaError_t me = cudaMalloc(&w.ptr, need);
    if (me == cudaSuccess) me = cudaMemset(w.ptr, 0, need);  // progress counters start at 0
    if (me != cudaSuccess) {
      if (w.ptr) cudaFree(w.ptr);
      w.ptr = nullptr;
      return cuda_fail(me);
    }
    w.bytes = need;
  }
  *out = w.ptr;
  *bytes = w.bytes;
  return MOE_OK;
}

// Fixed scratch for moe_switchglu_forward_static: one copy per device, in the
// module's global memory (zero at module load), so that entry never allocates.
// 4 MiB covers T*k <= 128 pairs at hidden 4096 / inter 2048 (2,629,632 bytes
// at T=16, k=8) and every smaller layer.
constexpr size_t kStaticScratchBytes = MOE_STATIC_SCRATCH_BYTES;
static_assert(kSyncWords == 1539, "the header states the counter region as 4*1539 bytes");
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];
void* g_static_ptr[kMaxDevices] = {};

// Device address of g_static_scratch for the current device: looked up once
// per device (cudaGetSymbolAddress, with that device current), then cached.
moe_status static_scratch(void** out) {
  int dev = 0;
  const cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return cuda_fail(ge);
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    if (!p) return MOE_ERR_CUDA;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace qeg

using namespace qeg;

extern "C" {

const char* moe_last_error(void) { return g_last_error; }

const char* moe_status_str(int s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_INDEX: return "MOE_ERR_DEVICE_INDEX";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    default: return "MOE_ERR_UNKNOWN";
  }
}

size_t moe_workspace_size(int T, int k, int E, int hidden, int inter) {
  if (!shape_ok(T, k, E, hidden, inter)) return 0;
  return ws_layout(T, k, E, hidden, inter).total;
}

moe_status moe_workspace_layout(int T, int k, int E, int hidden, int inter, size_t out[8]) {
  if (!out || !shape_ok(T, k, E, hidden, inter)) return MOE_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(T, k, E, hidden, inter);
  out[0] = w.barrier;
  out[1] = w.num_unique;
  out[2] = w.unique;
  out[3] = w.offsets;
  out[4] = w.pair_list;
  out[5] = w.h;
  out[6] = w.y;
  out[7] = w.total;
  return MOE_OK;
}

int moe_select_path(int T, int k, int E, int hidden, int inter) {
  return select_path(T, k, E, hidden, inter);
}

int moe_select_path_mxfp4(int T, int k, int E, int hidden, int inter) {
  return select_path(T, k, E, hidden, inter, kFmtMx);
}

size_t moe_workspace_size_mxfp4(int T, int k, int E, int hidden, int inter) {
  if (!shape_ok(T, k, E, hidden, inter)) return 0;
  return ws_layout(T, k, E, hidden, inter, kFmtMx).total;
}

moe_status moe_router_topk(const float* logits, int T, int E, int k, int renormalize,
                           int32_t* topk_idx, float* topk_w, void* stream) {
  if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (T <= 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > kRouterMaxE || k > kRouterMaxK || (long long)T * k > MOE_MAX_PAIRS)
    return MOE_ERR_UNSUPPORTED;
  if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
    return MOE_ERR_UNSUPPORTED;
  const int grid = (T + kRouterWarps - 1) / kRouterWarps;
  router_topk_kernel<<<grid, 32 * kRouterWarps, 0, (cudaStream_t)stream>>>(
      logits, T, E, k, renormalize ? 1 : 0, topk_idx, topk_w);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_route_union(const int32_t* topk_idx, int T, int k, int E, int32_t* unique,
                           int32_t* offsets, int32_t* pair_list, int32_t* num_unique,
                           void* stream) {
  if (!topk_idx || !unique || !offsets || !pair_list || !num_unique) return MOE_ERR_INVALID_ARG;
  if (T <= 0 || k <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
  if ((long long)T * k > MOE_MAX_PAIRS || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (!aligned(topk_idx, 4) || !aligned(unique, 4) || !aligned(offsets, 4) ||
      !aligned(pair_list, 4) || !aligned(num_unique, 4))
    return MOE_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  if (moe_status s = device_info(&d)) return s;
  const size_t smem = route_union_smem_bytes(E);
  if (smem > (size_t)d->dyn_smem[1]) return MOE_ERR_UNSUPPORTED;
  route_union_kernel<<<1, 32 * kUnionWarps, smem, (cudaStream_t)stream>>>(
      topk_idx, T * k, E, unique, offsets, pair_list, num_unique);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_switchglu_forward_ws(const uint16_t* x, const int32_t* topk_idx,
                                    const float* topk_w, const uint32_t* wg_q,
                                    const uint16_t* wg_s, const uint16_t* wg_b,
                                    const uint32_t* wu_q, const uint16_t* wu_s,
                                    const uint16_t* wu_b, const uint32_t* wd_q,
                                    const uint16_t* wd_s, const uint16_t* wd_b, int T, int k,
                                    int E, int hidden, int inter, uint16_t* out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!x || !topk_idx || !topk_w || !wg_q || !wg_s || !wg_b || !wu_q || !wu_s || !wu_b ||
      !wd_q || !wd_s || !wd_b || !out || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, k, E, hidden, inter)) return MOE_ERR_INVALID_ARG;
  const void* a16[] = {x, wg_q, wg_s, wg_b, wu_q, wu_s, wu_b, wd_q, wd_s, wd_b, out, workspace};
  for (const void* p : a16)
    if (!aligned(p, 16)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_UNSUPPORTED;
  const int path = select_path(T, k, E, hidden, inter);
  if (path == 0) return MOE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(T, k, E, hidden, inter).total) return MOE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if (moe_status s = device_info(&d)) return s;
  moe_status why = MOE_OK;
  unsigned char* wsp = static_cast<unsigned char*>(workspace);
  const cudaError_t e =
      path == 1 ? launch_layer<kFmtAffine>(x, topk_idx, topk_w, wg_q, wg_s, wg_b, wu_q, wu_s,
                                           wu_b, wd_q, wd_s, wd_b, T, k, E, hidden, inter, out,
                                           wsp, *d, (cudaStream_t)stream, &why)
                : launch_grouped<kFmtAffine>(x, topk_idx, topk_w, wg_q, wg_s, wg_b, wu_q, wu_s,
                                             wu_b, wd_q, wd_s, wd_b, T, k, E, hidden, inter, out,
                                             wsp, *d, (cudaStream_t)stream, &why);
  if (why != MOE_OK) return why;
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_switchglu_forward(const uint16_t* x, const int32_t* topk_idx, const float* topk_w,
                                 const uint32_t* wg_q, const uint16_t* wg_s,
                                 const uint16_t* wg_b, const uint32_t* wu_q,
                                 const uint16_t* wu_s, const uint16_t* wu_b,
                                 const uint32_t* wd_q, const uint16_t* wd_s,
                                 const uint16_t* wd_b, int T, int k, int E, int hidden,
                                 int inter, uint16_t* out, void* stream) {
  if (!shape_ok(T, k, E, hidden, inter)) return MOE_ERR_INVALID_ARG;
  void* ws = nullptr;
  size_t bytes = 0;
  if (moe_status s = owned_workspace(T, k, E, hidden, inter, kFmtAffine, stream, &ws, &bytes))
    return s;
  return moe_switchglu_forward_ws(x, topk_idx, topk_w, wg_q, wg_s, wg_b, wu_q, wu_s, wu_b, wd_q,
                                  wd_s, wd_b, T, k, E, hidden, inter, out, ws, bytes, stream);
}

moe_status moe_switchglu_forward_routed_ws(
    const uint16_t* x, const float* logits, int renormalize, const uint32_t* wg_q,
    const uint16_t* wg_s, const uint16_t* wg_b, const uint32_t* wu_q, const uint16_t* wu_s,
    const uint16_t* wu_b, const uint32_t* wd_q, const uint16_t* wd_s, const uint16_t* wd_b, int T,
    int k, int E, int hidden, int inter, uint16_t* out, int32_t* topk_idx, float* topk_w,
    void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !logits || !wg_q || !wg_s || !wg_b || !wu_q || !wu_s || !wu_b || !wd_q || !wd_s ||
      !wd_b || !out || !topk_idx || !topk_w || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, k, E, hidden, inter) || k > E) return MOE_ERR_INVALID_ARG;
  if (E > kRouterMaxE || k > kRouterMaxK) return MOE_ERR_UNSUPPORTED;
  const void* a16[] = {x, wg_q, wg_s, wg_b, wu_q, wu_s, wu_b, wd_q, wd_s, wd_b, out, workspace};
  for (const void* p : a16)
    if (!aligned(p, 16)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
    return MOE_ERR_UNSUPPORTED;
  const int path = select_path(T, k, E, hidden, inter, kFmtAffine, true);
  if (path == 0) return MOE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(T, k, E, hidden, inter).total) return MOE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if (moe_status s = device_info(&d)) return s;
  const cudaStream_t st = (cudaStream_t)stream;
  moe_status why = MOE_OK;
  cudaError_t e;
  if (path == 1) {
    e = launch_layer<kFmtAffine>(x, nullptr, nullptr, wg_q, wg_s, wg_b, wu_q, wu_s, wu_b, wd_q,
                                 wd_s, wd_b, T, k, E, hidden, inter, out,
                                 static_cast<unsigned char*>(workspace), *d, st, &why, logits,
                                 renormalize ? 1 : 0, topk_idx, topk_w);
  } else {
    // the grouped path takes the picks from the router kernel, then its five launches
    router_topk_kernel<<<(T + kRouterWarps - 1) / kRouterWarps, 32 * kRouterWarps, 0, st>>>(
        logits, T, E, k, renormalize ? 1 : 0, topk_idx, topk_w);
    e = cudaGetLastError();
    if (e == cudaSuccess)
      e = launch_grouped<kFmtAffine>(x, topk_idx, topk_w, wg_q, wg_s, wg_b, wu_q, wu_s, wu_b,
                                     wd_q, wd_s, wd_b, T, k, E, hidden, inter, out,
                                     static_cast<unsigned char*>(workspace), *d, st, &why);
  }
  if (why != MOE_OK) return why;
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_switchglu_forward_routed(const uint16_t* x, const float* logits, int renormalize,
                                        const uint32_t* wg_q, const uint16_t* wg_s,
                                        const uint16_t* wg_b, const uint32_t* wu_q,
                                        const uint16_t* wu_s, const uint16_t* wu_b,
                                        const uint32_t* wd_q, const uint16_t* wd_s,
                                        const uint16_t* wd_b, int T, int k, int E, int hidden,
                                        int inter, uint16_t* out, int32_t* topk_idx,
                                        float* topk_w, void* stream) {
  if (!shape_ok(T, k, E, hidden, inter)) return MOE_ERR_INVALID_ARG;
  void* ws = nullptr;
  size_t bytes = 0;
  if (moe_status s = owned_workspace(T, k, E, hidden, inter, kFmtAffine, stream, &ws, &bytes))
    return s;
  return moe_switchglu_forward_routed_ws(x, logits, renormalize, wg_q, wg_s, wg_b, wu_q, wu_s,
                                         wu_b, wd_q, wd_s, wd_b, T, k, E, hidden, inter, out,
                                         topk_idx, topk_w, ws, bytes, stream);
}

moe_status moe_switchglu_forward_static(const uint16_t* x, const int32_t* topk_idx,
                                        const float* topk_w, const uint32_t* wg_q,
                                        const uint16_t* wg_s, const uint16_t* wg_b,
                                        const uint32_t* wu_q, const uint16_t* wu_s,
                                        const uint16_t* wu_b, const uint32_t* wd_q,
                                        const uint16_t* wd_s, const uint16_t* wd_b, int T, int k,
                                        int E, int hidden, int inter, uint16_t* out,
                                        void* stream) {
  if (!shape_ok(T, k, E, hidden, inter)) return MOE_ERR_INVALID_ARG;
  const size_t need = ws_layout(T, k, E, hidden, inter).total;
  if (need > kStaticScratchBytes) {
    g_last_error = "moe_switchglu_forward_static: this shape needs more scratch than the "
                   "fixed 4 MiB (4194304 bytes); use moe_switchglu_forward_ws";
    return MOE_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (moe_status s = static_scratch(&scratch)) return s;
  // The progress counters must be zero when the kernel starts; a call clears
  // them again on the caller's stream (ordered after any earlier call there),
  // so a call that ended with a device error leaves no stale counts behind.
  const cudaError_t me = cudaMemsetAsync(scratch, 0, 4 * kSyncWords, (cudaStream_t)stream);
  if (me != cudaSuccess) return cuda_fail(me);
  return moe_switchglu_forward_ws(x, topk_idx, topk_w, wg_q, wg_s, wg_b, wu_q, wu_s, wu_b, wd_q,
                                  wd_s, wd_b, T, k, E, hidden, inter, out, scratch,
                                  kStaticScratchBytes, stream);
}

moe_status moe_switchglu_forward_mxfp4_ws(const uint16_t* x, const int32_t* topk_idx,
                                          const float* topk_w, const uint32_t* wg_q,
                                          const uint8_t* wg_e, const uint32_t* wu_q,
                                          const uint8_t* wu_e, const uint32_t* wd_q,
                                          const uint8_t* wd_e, int T, int k, int E, int hidden,
                                          int inter, uint16_t* out, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  if (!x || !topk_idx || !topk_w || !wg_q || !wg_e || !wu_q || !wu_e || !wd_q || !wd_e ||
      !out || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, k, E, hidden, inter)) return MOE_ERR_INVALID_ARG;
  const void* a16[] = {x, wg_q, wg_e, wu_q, wu_e, wd_q, wd_e, out, workspace};
  for (const void* p : a16)
    if (!aligned(p, 16)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(topk_idx, 4) || !aligned(topk_w, 4)) return MOE_ERR_UNSUPPORTED;
  const int path = select_path(T, k, E, hidden, inter, kFmtMx);
  if (path == 0) return MOE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(T, k, E, hidden, inter, kFmtMx).total) return MOE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if (moe_status s = device_info(&d)) return s;
  moe_status why = MOE_OK;
  // the e8m0 scale arrays travel in the scale slots; the format has no biases
  const uint16_t* ge = reinterpret_cast<const uint16_t*>(wg_e);
  const uint16_t* ue = reinterpret_cast<const uint16_t*>(wu_e);
  const uint16_t* de = reinterpret_cast<const uint16_t*>(wd_e);
  unsigned char* wsp = static_cast<unsigned char*>(workspace);
  const cudaError_t e =
      path == 1 ? launch_layer<kFmtMx>(x, topk_idx, topk_w, wg_q, ge, nullptr, wu_q, ue, nullptr,
                                       wd_q, de, nullptr, T, k, E, hidden, inter, out, wsp, *d,
                                       (cudaStream_t)stream, &why)
                : launch_grouped<kFmtMx>(x, topk_idx, topk_w, wg_q, ge, nullptr, wu_q, ue,
                                         nullptr, wd_q, de, nullptr, T, k, E, hidden, inter, out,
                                         wsp, *d, (cudaStream_t)stream, &why);
  if (why != MOE_OK) return why;
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_switchglu_forward_mxfp4(const uint16_t* x, const int32_t* topk_idx,
                                       const float* topk_w, const uint32_t* wg_q,
                                       const uint8_t* wg_e, const uint32_t* wu_q,
                                       const uint8_t* wu_e, const uint32_t* wd_q,
                                       const uint8_t* wd_e, int T, int k, int E, int hidden,
                                       int inter, uint16_t* out, void* stream) {
  if (!shape_ok(T, k, E, hidden, inter)) return MOE_ERR_INVALID_ARG;
  void* ws = nullptr;
  size_t bytes = 0;
  if (moe_status s = owned_workspace(T, k, E, hidden, inter, kFmtMx, stream, &ws, &bytes))
    return s;
  return moe_switchglu_forward_mxfp4_ws(x, topk_idx, topk_w, wg_q, wg_e, wu_q, wu_e, wd_q, wd_e,
                                        T, k, E, hidden, inter, out, ws, bytes, stream);
}

moe_status moe_set_wait_limit_ns(unsigned long long ns) {
  const unsigned long long v = ns == 0 ? kWaitLimitNs : (ns < 1000ull ? 1000ull : ns);
  if (v > kWaitLimitNs) return MOE_ERR_INVALID_ARG;
  const cudaError_t e = cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

moe_status moe_read_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e);
  if (word) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (word & kErrTimeout) {
    // A call that gave up on a bounded wait may have left its progress counters
    // non-zero.  The stream is idle now, so clear those of the workspace this
    // library owns on the current device (moe_switchglu_forward's); a caller-owned
    // workspace is the caller's to clear, and the static scratch is cleared by
    // every call of moe_switchglu_forward_static.
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev >= 0 && dev < kMaxDevices) {
      std::lock_guard<std::mutex> lock(g_mu);
      if (g_ws[dev].ptr) {
        e = cudaMemset(g_ws[dev].ptr, 0, 4 * kSyncWords);
        if (e != cudaSuccess) return cuda_fail(e);
      }
    }
    return MOE_ERR_TIMEOUT;
  }
  if (word & kErrExpertIndex) return MOE_ERR_DEVICE_INDEX;
  return MOE_OK;
}

}  // extern "C"
