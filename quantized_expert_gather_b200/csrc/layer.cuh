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
//             to `seg` of its pairs; the CTAs convert the window's x rows to
//             block fixed point in the workspace, together;
//   phase A   gate+up over items of 32 rows (segment, rows of Wg and Wu):
//               h = bf16(silu(bf16(Wg x)) * bf16(Wu x))
//             (the one-pass epilogue of "Apple7/8 MoE gate and up in one decode
//             pass", splash PR 45, "What changed"); the item's 32 h values per
//             pair are one fixed-point chunk, converted at the item's end;
//   phase B   down over items of rows_b rows of Wd: y = Wd h per pair, fp32.
//             A segment's phase-B items start once every phase-A item of that
//             segment has published (counter hdone[seg]);
//   combine   out[t] = bf16(sum_j w[t,j] * y[t,j]) per block of rows_b output
//             rows, by CTA (row block mod grid) once every segment of the row
//             block has published (counter ydone[rb]).
// Work items are taken from one list (all phase-A items, segment-major, then all
// phase-B items) through a counter in the workspace, so CTAs stay balanced and a
// phase-B item's h is normally complete long before the item is taken.  An
// expert with more than `seg` pairs in the window forms several segments and is
// streamed once per segment.  Every spin on a counter or barrier is bounded
// (common.cuh); the counters are zero again when the kernel ends.
//
// Warps: 8 compute warps and one producer warp.  The producer takes work items,
// issues every bulk copy (weights into a ring of stages, activation rows into
// one of two activation buffers) and publishes finished items; the compute warps
// wait only on mbarriers and, at the end of a phase-A item, on a named barrier.
//
// Compute: each warp owns whole rows (phase A: one row of Wg and the same row
// of Wu; phase B: up to 4 rows of Wd) over the full input width.  Lane l takes
// the 32-column chunks l, l+32, ... of its rows, so one lane chunk sits inside
// one quantisation group (64 columns):
//     partial = s * sum_c q_c x_c + b * sum_c x_c.
// Activations are 16-bit block fixed point (one exponent per 32-column chunk,
// see below), so that sum_c q_c x_c is an exact integer dot product of the 4-bit
// codes with the activation's two bytes (dp4a), scaled once per chunk.  A warp
// reduces its rows over its lanes once per block.
#pragma once

#include "common.cuh"
#include "union.cuh"

namespace qeg {

// Bank formats.  kFmtAffine: 4-bit codes, bf16 scale and bias per 64 columns
// (w = s q + b).  kFmtMx: mxfp4, e2m1 codes and one e8m0 scale per 32 columns
// (w = e2m1(q) 2^(e - 127)).  Codes are packed alike in both.
constexpr int kFmtAffine = 0;
constexpr int kFmtMx = 1;

constexpr int kWarps = 8;                    // compute warps
constexpr int kConsumerThreads = 32 * kWarps;
constexpr int kThreads = kConsumerThreads + 64;  // + a producer warp and a helper warp
constexpr int kRowsA = kWarps;      // phase A: one row of gate and of up per warp per block
constexpr int kBlocksPerItemA = 4;  // phase-A item: 4 blocks = 32 rows = one h chunk
constexpr int kBlocksPerItemB = 2;  // phase-B item: row blocks
constexpr int kMaxRowsPerWarpB = 4; // phase B: rows of Wd per warp per block
constexpr int kMaxStages = 4;       // ring depth (fewer when shared memory is short)
constexpr int kNT = 4;              // pairs per segment (upper bound)
constexpr int kMaxPairsFused = 1024;
constexpr unsigned kSegActBytes = 36 * 1024;  // one activation buffer (a segment's rows)
constexpr int kItemRing = 16;       // items between compute and publication
// Dynamic shared memory the kernel may plan for on B200 (227 KB per block, less a
// margin for its static shared memory).
constexpr size_t kSmemBudget = 232448 - 1024;

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Bytes of one activation row in the fixed-point layout (digits, then per-chunk
// scale and sum; see "activations and codes"), R rounds of 32 chunks.
__host__ __device__ constexpr unsigned act_bytes(int R) { return 2304u * (unsigned)R; }
__host__ __device__ constexpr unsigned act_digit_bytes(int R) { return 2048u * (unsigned)R; }

// ---------------------------------------------------------------- geometry ---
struct LayerGeom {
  int fmt;                 // kFmtAffine or kFmtMx
  int rounds_a, rounds_b;  // 32-column chunks per lane per row (>= H/1024, I/1024; 1, 2, 4, 6, 8)
  int rows_b;              // phase B rows per block (multiple of kWarps, <= 32)
  int seg;                 // pairs per segment (<= kNT)
  int stages;              // ring depth (<= kMaxStages)
  unsigned a_q, a_sb, a_mat, a_bytes;  // phase A block: per matrix codes / scale (or bias) bytes
  unsigned b_q, b_sb, b_bytes;         // phase B full block
  unsigned stage_bytes;
  unsigned act_buf;        // one activation buffer: seg rows of the wider layout
};

// Chunk rounds for a row of D columns: ceil(D / 1024), rounded up to 1, 2, 4, 6 or 8.
__host__ __device__ inline int chunk_rounds(int D) {
  const int r = (D + 1023) / 1024;
  return r <= 2 ? r : (r <= 4 ? 4 : (r <= 6 ? 6 : 8));
}

__host__ __device__ inline LayerGeom layer_geom(int H, int I, int fmt = kFmtAffine) {
  LayerGeom g;
  g.fmt = fmt;
  g.rounds_a = chunk_rounds(H);
  g.rounds_b = chunk_rounds(I);
  int rb = (16 * H / I) / kWarps * kWarps;  // about one phase-A stage worth of Wd rows
  if (rb < kWarps) rb = kWarps;
  if (rb > kWarps * kMaxRowsPerWarpB) rb = kWarps * kMaxRowsPerWarpB;
  g.rows_b = rb;
  const int rmax = g.rounds_a > g.rounds_b ? g.rounds_a : g.rounds_b;
  int s = (int)(kSegActBytes / act_bytes(rmax));
  g.seg = s > kNT ? kNT : s;
  g.stages = kMaxStages;
  g.a_q = kRowsA * H / 2;
  // scales: bf16 per 64 columns (affine) or one e8m0 byte per 32 (mx), H/32 bytes a
  // row either way; the affine format adds as many bytes of biases
  const int nsb = fmt == kFmtMx ? 1 : 2;
  g.a_sb = kRowsA * H / 32;
  g.a_mat = g.a_q + nsb * g.a_sb;
  g.a_bytes = 2 * g.a_mat;
  g.b_q = g.rows_b * I / 2;
  g.b_sb = g.rows_b * I / 32;
  g.b_bytes = g.b_q + nsb * g.b_sb;
  g.stage_bytes = (unsigned)align_up(g.a_bytes > g.b_bytes ? g.a_bytes : g.b_bytes, 128);
  g.act_buf = (unsigned)align_up((size_t)(g.seg > 0 ? g.seg : 1) * act_bytes(rmax), 128);
  return g;
}

struct LayerSmem {
  size_t stages, act, hscr, cnt, rank, unique, offsets, pair_list, pos_of, seg_slot, seg_pos,
      seg_nt, total;
};
__host__ __device__ inline LayerSmem layer_smem(const LayerGeom& g, int E, int P, int H, int I) {
  LayerSmem s;
  const int m = (E < P ? E : P) > 0 ? (E < P ? E : P) : 1;
  s.stages = 0;
  s.act = align_up((size_t)g.stages * g.stage_bytes, 128);    // two activation buffers
  s.hscr = s.act + 2 * (size_t)g.act_buf;  // bf16 h of phase-A items, per item ring slot
  s.cnt = align_up(s.hscr + sizeof(uint16_t) * kItemRing * kNT * 32, 16);
  s.rank = align_up(s.cnt + sizeof(int) * E, 16);
  s.unique = align_up(s.rank + sizeof(int) * P, 16);
  s.offsets = align_up(s.unique + sizeof(int) * m, 16);
  s.pair_list = align_up(s.offsets + sizeof(int) * (m + 1), 16);
  s.pos_of = align_up(s.pair_list + sizeof(int) * P, 16);
  // segments: at most P of them
  s.seg_slot = align_up(s.pos_of + sizeof(int) * P, 16);
  s.seg_pos = align_up(s.seg_slot + sizeof(int) * P, 16);
  s.seg_nt = align_up(s.seg_pos + sizeof(int) * P, 16);
  s.total = align_up(s.seg_nt + sizeof(int) * P, 16);
  return s;
}

// Deepest ring (kMaxStages down to 2) whose shared memory fits in `budget` bytes;
// false if none does.
__host__ __device__ inline bool fit_stages(LayerGeom& g, int E, int P, int H, int I,
                                           size_t budget) {
  for (int st = kMaxStages; st >= 2; --st) {
    g.stages = st;
    if (layer_smem(g, E, P, H, I).total <= budget) return true;
  }
  return false;
}

// Workspace counters (unsigned), a region of fixed size at the start of every
// workspace so that calls of different shapes never see each other's data there:
// [0] CTAs finished, [1, 1+kMaxPairsFused) hdone per segment, then ydone per
// phase-B row block (at most kMaxRowBlocks), then the work-item counter and the
// count of CTAs that have converted their share of x.
constexpr int kMaxRowBlocks = 4096 / kWarps;
constexpr size_t kSyncWords = 1 + kMaxPairsFused + kMaxRowBlocks + 2;
constexpr size_t kSyncWorkItem = 1 + kMaxPairsFused + kMaxRowBlocks;
constexpr size_t kSyncXDone = kSyncWorkItem + 1;

// -------------------------------------------------------------- arguments ---
struct LayerArgs {
  const uint16_t* x;  // [T, H] bf16
  const int* idx;     // [T, k]
  const float* w;     // [T, k]
  const uint32_t *gq, *uq, *dq;
  const uint16_t *gs, *gb, *us, *ub, *ds, *db;
  uint16_t* h;        // workspace [P, I] bf16, rows in pair_list order
  float* y;           // workspace [P, H] fp32, rows in pair_list order
  unsigned char* xg;  // workspace: x rows in the fixed-point layout, [T] x act_bytes(rounds_a)
  unsigned char* hq;  // workspace: h rows in the fixed-point layout, [P] x act_bytes(rounds_b)
  unsigned* sync;     // workspace counters (kSyncWords)
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
// Layout of one activation row (a token's x or a pair's h) of D columns, R rounds
// (R a power of two >= D / 1024), in act_bytes(R) = 2304 R bytes: for chunk
// ch = i * 32 + l (i < R, l < 32) the uint4 at index (i * 4 + m) * 32 + l covers
// columns 32 ch + 8m .. +7 as
//   .x = low bytes of columns 8m+0,2,4,6   .y = low bytes of 8m+1,3,5,7
//   .z = high bytes of columns 8m+0,2,4,6  .w = high bytes of 8m+1,3,5,7
// followed (at byte 2048 R) by float2 sc[ch] = (2^(e - 14), sum of the chunk's 32
// values).  The same layout serves in global memory (converted once per call) and
// in shared memory (copied per work item).
constexpr uint32_t kNibbleBytes = 0x0F0F0F0Fu;

__device__ __forceinline__ int dp4a_lo(uint32_t q, uint32_t d, int c) {
  return static_cast<int>(__dp4a(q, d, static_cast<unsigned>(c)));
}
__device__ __forceinline__ int dp4a_hi(uint32_t q, uint32_t d, int c) {
  return __dp4a(static_cast<int>(q), static_cast<int>(d), c);
}


// Chunk (round i, lane) of an activation row into registers.
__device__ __forceinline__ void load_xq(const unsigned char* row, int i, int lane,
                                        uint4 (&d)[4]) {
  const uint4* p = reinterpret_cast<const uint4*>(row) + (i * 4) * 32 + lane;
#pragma unroll
  for (int m = 0; m < 4; ++m) d[m] = p[m * 32];
}
__device__ __forceinline__ float2 load_sc(const unsigned char* row, int R, int ch) {
  return reinterpret_cast<const float2*>(row + act_digit_bytes(R))[ch];
}

// sum_c q_c v_c over one chunk (4 code words, 4 activation uint4), exact.  Four
// partial sums keep the dp4a dependency chains short.
__device__ __forceinline__ int chunk_dot(const uint32_t (&qs)[8], const uint4 (&x)[4]) {
  int lo0 = 0, lo1 = 0, hi0 = 0, hi1 = 0;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint4 d = x[m];
    lo0 = dp4a_lo(qs[2 * m], d.x, lo0);
    lo1 = dp4a_lo(qs[2 * m + 1], d.y, lo1);
    hi0 = dp4a_hi(qs[2 * m], d.z, hi0);
    hi1 = dp4a_hi(qs[2 * m + 1], d.w, hi1);
  }
  return (hi0 + hi1) * 256 + (lo0 + lo1);  // |.| < 2^24: exact in fp32
}

// The 32 codes of a uint4, split as described above (affine format).
__device__ __forceinline__ void split_codes(const uint4 v, uint32_t (&qs)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    qs[2 * m] = w[m] & kNibbleBytes;
    qs[2 * m + 1] = (w[m] >> 4) & kNibbleBytes;
  }
}

// mxfp4 codes as bytes for dp4a.  An e2m1 code (sign bit 3, magnitude index bits
// 2..0 for 0, 0.5, 1, 1.5, 2, 3, 4, 6) becomes q' = 2 e2m1(q) + 12, an integer in
// [0, 24], so that  e2m1(q) = (q' - 12) / 2  and a chunk's sum is
// (sum q' v - 12 sum v) / 2.  Two byte lookups (prmt: four selectors from the 16
// low bits, each picking one of 8 table bytes; a selector with bit 3 set returns
// the sign fill of its byte, 0 for these tables) give the values of the positive
// codes and of the negative ones, each 0 where the other applies.  Bytes 0..3 of
// qs[2m] are codes 0..3 of word m (columns 8m .. 8m+3), bytes of qs[2m+1] codes
// 4..7: consecutive columns, the activation layout of this format.
constexpr uint32_t kMxPos0 = 0x0F0E0D0Cu, kMxPos1 = 0x18141210u;  // 12 + 2 * (0 .. 6)
constexpr uint32_t kMxNeg0 = 0x090A0B0Cu, kMxNeg1 = 0x00040608u;  // 12 - 2 * (0 .. 6)
// PTX prmt in its default mode (a selector's bit 3 asks for the sign fill).
__device__ __forceinline__ uint32_t prmt_sign(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t mx_bytes(uint32_t sel) {
  return prmt_sign(kMxPos0, kMxPos1, sel) | prmt_sign(kMxNeg0, kMxNeg1, sel ^ 0x8888u);
}
__device__ __forceinline__ void split_codes_mx(const uint4 v, uint32_t (&qs)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    qs[2 * m] = mx_bytes(w[m]);
    qs[2 * m + 1] = mx_bytes(w[m] >> 16);
  }
}

template <int F>
__device__ __forceinline__ void split_codes_f(const uint4 v, uint32_t (&qs)[8]) {
  if constexpr (F == kFmtMx) split_codes_mx(v, qs);
  else split_codes(v, qs);
}

// 2^(e - 128) for an e8m0 byte e (half the mxfp4 block scale 2^(e - 127)); NaN for 255.
__device__ __forceinline__ float mx_half_scale(uint32_t e) {
  if (e >= 2u && e < 255u) return __uint_as_float((e - 1u) << 23);
  if (e == 255u) return __uint_as_float(0x7fc00000u);
  return __uint_as_float(0x00400000u >> (1u - e));  // 2^-127, 2^-128: subnormal
}

// Scale and bias applied to a chunk's exact sum:  partial = sv * 2^(e-14) * dot +
// bv * sum x.  Affine: the group's (s, b), group ch / 2.  mxfp4: (2^(e-128),
// -12 * 2^(e-128)) from the chunk's own e8m0 byte (see mx_bytes).
template <int F>
__device__ __forceinline__ float2 chunk_sb(const uint16_t* s, const uint16_t* b, int ch) {
  if constexpr (F == kFmtMx) {
    const float h = mx_half_scale(reinterpret_cast<const uint8_t*>(s)[ch]);
    return make_float2(h, -12.0f * h);
  } else {
    return make_float2(bf16_bits_to_float(s[ch >> 1]), bf16_bits_to_float(b[ch >> 1]));
  }
}

// One thread's quarter of a chunk: the 8 bf16 values of columns 8m .. 8m+7 (in v)
// become this thread's uint4 of the layout above; the 4 threads of a chunk are
// consecutive lanes (group mask gmask).  Returns the chunk's (scale, sum) in every
// thread of the group.
template <int F>
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
    // affine: k even -> .x/.z, odd -> .y/.w, byte k / 2; mxfp4: k < 4 -> .x/.z,
    // else .y/.w, byte k % 4 (the orders the two code splits produce)
    const int wsel = F == kFmtMx ? (k >> 2) : (k & 1);
    const int pos = F == kFmtMx ? (k & 3) * 8 : (k >> 1) * 8;
    lo[wsel] |= (static_cast<uint32_t>(val) & 0xffu) << pos;
    hi[wsel] |= ((static_cast<uint32_t>(val) >> 8) & 0xffu) << pos;
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

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
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
// Phase A: this warp's row of Wg and of Wu, NT pairs (activation rows act + t *
// stride), R rounds of 32-column chunks (chunks past H/32 skipped); returns (G, U)
// for t < NT in every lane.  Per chunk (inside one quantisation group):
// s * 2^(e-14) * sum q v + b * sum x.
template <int NT, int R, int F>
__device__ __forceinline__ void rows_a(const unsigned char* bg_q, const uint16_t* bg_s,
                                       const uint16_t* bg_b, const unsigned char* bu_q,
                                       const uint16_t* bu_s, const uint16_t* bu_b, int H,
                                       const unsigned char* act, unsigned stride, int lane,
                                       float (&G)[kNT], float (&U)[kNT]) {
  float ag[NT], au[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) ag[t] = au[t] = 0.f;
  const int nch = H / 32;
  constexpr int kRoundUnroll = NT == 1 ? 2 : 1;  // one pair: two chunks in flight
#pragma unroll kRoundUnroll
  for (int i = 0; i < R; ++i) {
    const int ch = i * 32 + lane;
    if (ch < nch) {
      uint32_t qg[8], qu[8];
      split_codes_f<F>(*reinterpret_cast<const uint4*>(bg_q + ch * 16), qg);
      split_codes_f<F>(*reinterpret_cast<const uint4*>(bu_q + ch * 16), qu);
      const float2 sbg = chunk_sb<F>(bg_s, bg_b, ch), sbu = chunk_sb<F>(bu_s, bu_b, ch);
      const float sg = sbg.x, bgv = sbg.y, su = sbu.x, buv = sbu.y;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const unsigned char* row = act + t * stride;
        uint4 xd[4];
        load_xq(row, i, lane, xd);
        const float2 sc = load_sc(row, R, ch);
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
template <int NT, int R, int F>
__device__ __forceinline__ float rows_b(const unsigned char* bq, const uint16_t* bs,
                                        const uint16_t* bb, int row0, int nrows, int I,
                                        const unsigned char* act, unsigned stride, int lane,
                                        int& vid) {
  constexpr int NP = (NT == 3) ? 4 : NT;
  constexpr int V = kMaxRowsPerWarpB * NP;
  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  const int nch = I / 32, qstride = I / 2, sstride = I / 64;
  constexpr int kRoundUnroll = NT == 1 ? 2 : 1;  // one pair: two chunks in flight
#pragma unroll kRoundUnroll
  for (int i = 0; i < R; ++i) {
    const int ch = i * 32 + lane;
    if (ch < nch) {
      float2 sc[NT];
      uint4 xd[NT][4];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const unsigned char* row = act + t * stride;
        sc[t] = load_sc(row, R, ch);
        load_xq(row, i, lane, xd[t]);
      }
#pragma unroll
      for (int q = 0; q < kMaxRowsPerWarpB; ++q) {
        const int r = row0 + kWarps * q;
        if (r < nrows) {
          uint32_t qs[8];
          split_codes_f<F>(*reinterpret_cast<const uint4*>(bq + (size_t)r * qstride + ch * 16), qs);
          // a row's scales: I/64 bf16 (affine) or I/32 bytes (mxfp4), I/32 bytes either way
          const float2 sb = chunk_sb<F>(bs + r * sstride, bb + r * sstride, ch);
          const float sv = sb.x, bv = sb.y;
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

template <int NT, int F>
__device__ __forceinline__ void dispatch_a(int R, const unsigned char* bgq, const uint16_t* bgs,
                                           const uint16_t* bgb, const unsigned char* buq,
                                           const uint16_t* bus, const uint16_t* bub, int H,
                                           const unsigned char* act, unsigned stride, int lane,
                                           float (&G)[kNT], float (&U)[kNT]) {
  if (R == 1) rows_a<NT, 1, F>(bgq, bgs, bgb, buq, bus, bub, H, act, stride, lane, G, U);
  else if (R == 2) rows_a<NT, 2, F>(bgq, bgs, bgb, buq, bus, bub, H, act, stride, lane, G, U);
  else if (R == 4) rows_a<NT, 4, F>(bgq, bgs, bgb, buq, bus, bub, H, act, stride, lane, G, U);
  else if (R == 6) rows_a<NT, 6, F>(bgq, bgs, bgb, buq, bus, bub, H, act, stride, lane, G, U);
  else rows_a<NT, 8, F>(bgq, bgs, bgb, buq, bus, bub, H, act, stride, lane, G, U);
}

template <int NT, int F>
__device__ __forceinline__ float dispatch_b(int R, const unsigned char* bq, const uint16_t* bs,
                                            const uint16_t* bb, int row0, int nrows, int I,
                                            const unsigned char* act, unsigned stride, int lane,
                                            int& vid) {
  if (R == 1) return rows_b<NT, 1, F>(bq, bs, bb, row0, nrows, I, act, stride, lane, vid);
  if (R == 2) return rows_b<NT, 2, F>(bq, bs, bb, row0, nrows, I, act, stride, lane, vid);
  if (R == 4) return rows_b<NT, 4, F>(bq, bs, bb, row0, nrows, I, act, stride, lane, vid);
  if (R == 6) return rows_b<NT, 6, F>(bq, bs, bb, row0, nrows, I, act, stride, lane, vid);
  return rows_b<NT, 8, F>(bq, bs, bb, row0, nrows, I, act, stride, lane, vid);
}

// mbarrier phase test without suspending (for wait loops that do other work).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Order this thread's generic-proxy view of global memory (data other CTAs
// published and this thread acquired) before its following bulk copies.
__device__ __forceinline__ void fence_proxy_async_all() {
  asm volatile("fence.proxy.async;" ::: "memory");
}

// Lane 0's value of a condition, in every lane (keeps the producer warp's control
// flow uniform when lanes could read a changing value at different times).
__device__ __forceinline__ bool lane0(bool v) { return __shfl_sync(kFull, v ? 1 : 0, 0) != 0; }
__device__ __forceinline__ int lane0_int(int v) { return __shfl_sync(kFull, v, 0); }

// Ring-slot descriptor flags (slot_info[st].x) for the compute warps.
constexpr int kSlotEnd = 1;        // no more blocks
constexpr int kSlotPhaseB = 2;     // a phase-B block
constexpr int kSlotItemEnd = 4;    // last block of its work item
constexpr int kSlotActWait = 8;    // first block of an item whose activation rows were loaded
constexpr int kSlotActPar = 16;    // parity of that load's phase on act_full[ord % kItemRing]
constexpr int kSlotActShift = 8;   // bits 8..: byte offset / 128 of the item's activation rows

// 9 warps: 8 compute warps and one producer warp (see the top of this file).
template <int F>
__global__ void __maxnreg__(168) layer_kernel(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_u, s_nseg;
  __shared__ volatile int s_abort;
  // producer <-> helper: items recorded / published, activation loads queued / issued,
  // producer finished
  __shared__ volatile int s_nrec, s_pub, s_pend_tail, s_pend_head, s_prod_done;
  __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ __align__(8) uint64_t act_full[kItemRing], item_done[kItemRing];
  __shared__ unsigned long long reg_start[kItemRing];  // activation regions (producer)
  __shared__ int reg_last[kItemRing];
  __shared__ int4 item_info[kItemRing];  // per item ordinal: phase B, segment, first block, blocks
  __shared__ int4 pend[kItemRing];       // queued activation loads (producer)
  __shared__ int4 slot_info[kMaxStages];  // per ring slot: flags, segment, first row, item ordinal
  const LayerGeom& G = a.g;
  const int P = a.T * a.k;
  const int NS = G.stages;
  const LayerSmem L = layer_smem(G, a.E, P, a.H, a.I);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned* exit_cnt = a.sync;
  unsigned* hdone = a.sync + 1;
  unsigned* ydone = a.sync + 1 + kMaxPairsFused;
  unsigned* work_ctr = a.sync + kSyncWorkItem;
  unsigned* xdone = a.sync + kSyncXDone;
  const unsigned stride_a = act_bytes(G.rounds_a), stride_b = act_bytes(G.rounds_b);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    for (int i = 0; i < kItemRing; ++i) {
      mbar_init(&act_full[i], 1);
      mbar_init(&item_done[i], kWarps);
    }
    s_abort = 0;
    s_nrec = s_pub = s_pend_tail = s_pend_head = s_prod_done = 0;
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

  // ---- x rows in the fixed-point layout, converted by all CTAs together ----
  {
    const int nch = a.H / 32, R = G.rounds_a;
    const long long nq = (long long)a.T * nch * 4;  // quarters of 8 columns
    for (long long q = (long long)blockIdx.x * kThreads + threadIdx.x; q < nq + 0;
         q += (long long)gridDim.x * kThreads) {
      const int m = (int)(q & 3), tc = (int)(q >> 2), t = tc / nch, ch = tc % nch;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H + ch * 32 + m * 8));
      uint4 packed;
      const float2 sc = fixed_point_quarter<F>(v, 0xfu << (lane & ~3), packed);
      unsigned char* row = a.xg + (size_t)t * stride_a;
      reinterpret_cast<uint4*>(row)[((ch / 32) * 4 + m) * 32 + (ch % 32)] = packed;
      if (m == 0) reinterpret_cast<float2*>(row + act_digit_bytes(R))[ch] = sc;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    red_release_gpu(xdone, 1u);
  }
  const int u = s_u, nseg = s_nseg;
  const int n_valid = offs[u];
  for (int i = threadIdx.x; i < n_valid; i += kThreads) pos_of[plist[i]] = i;
  __syncthreads();

  if (blockIdx.x == 0 && warp == 1 && a.ex_u) {
    for (int i = lane; i < u; i += 32) a.ex_unique[i] = uniq[i];
    for (int i = lane; i <= u; i += 32) a.ex_offsets[i] = offs[i];
    for (int i = lane; i < P; i += 32) a.ex_pair_list[i] = plist[i];
    if (lane == 0) *a.ex_u = u;
  }

  const int bpe_a = a.I / kRowsA;                     // phase-A blocks per segment
  const int ipa = bpe_a / kBlocksPerItemA;            // phase-A items per segment
  const int bpe_b = (a.H + G.rows_b - 1) / G.rows_b;  // phase-B blocks per segment
  // phase-B items: kBlocksPerItemB blocks each, except in the last quarter of the
  // segments, where single blocks keep the CTAs' finishing times close
  const int ipb = (bpe_b + kBlocksPerItemB - 1) / kBlocksPerItemB;
  const int seg_fine = nseg - (nseg + 3) / 4;  // first segment with single-block items
  const int n_items_a = nseg * ipa;
  const int n_items_b2 = seg_fine * ipb;
  const int n_items = n_items_a + n_items_b2 + (nseg - seg_fine) * bpe_b;

  if (warp == kWarps + 1) {
    // ================================ helper warp ================================
    // Publishes finished items in order (converting each phase-A item's h chunk to
    // the fixed-point layout first) and issues the queued activation loads once what
    // they read is complete.  Every condition is lane 0's (uniform control flow).
    const uint16_t* hscr_p = reinterpret_cast<const uint16_t*>(smem + L.hscr);
    int pub = 0, ph = 0;  // items published; queued loads issued
    bool x_ready = false;
    unsigned long long t_prog = globaltimer();
    for (;;) {
      bool progressed = false;
      // ---- publish ----
      const int n_rec = lane0_int(s_nrec);
      __threadfence_block();  // item_info of the recorded items is read after the count
      int n = 0;
      while (pub + n < n_rec &&
             lane0(mbar_test(&item_done[(pub + n) % kItemRing], ((pub + n) / kItemRing) & 1)))
        ++n;
      if (n > 0) {
        // a phase-A item's 32 h rows per pair are one chunk of h (lanes 4t..4t+3: pair t)
        for (int i = 0; i < n; ++i) {
          const int4 ii = item_info[(pub + i) % kItemRing];
          if (ii.x != 0) continue;
          const int nt = seg_nt[ii.y], p0 = seg_pos[ii.y];
          if (lane < nt * 4) {
            const int t = lane >> 2, m = lane & 3;
            const uint4 v = *reinterpret_cast<const uint4*>(
                hscr_p + ((pub + i) % kItemRing) * (kNT * 32) + t * 32 + m * 8);
            uint4 packed;
            const float2 sc = fixed_point_quarter<F>(v, 0xfu << (lane & ~3), packed);
            const int ch = ii.z / (32 / kRowsA), R = G.rounds_b;  // h chunk of the item
            unsigned char* row = a.hq + (size_t)(p0 + t) * stride_b;
            reinterpret_cast<uint4*>(row)[((ch / 32) * 4 + m) * 32 + (ch % 32)] = packed;
            if (m == 0) reinterpret_cast<float2*>(row + act_digit_bytes(R))[ch] = sc;
          }
        }
        __syncwarp();  // the lanes' hq writes precede lane 0's release below
        // The compute warps' item_done arrivals released their stores at CTA scope and
        // the tests above acquired them; the device-scope release reductions pass them
        // on (causality order is transitive across the two scopes).
        if (lane == 0) {
          for (int i = 0; i < n; ++i) {
            const int4 ii = item_info[(pub + i) % kItemRing];
            if (ii.x == 0) {
              red_release_gpu(&hdone[ii.y], (unsigned)ii.w);
            } else {
              for (int r = 0; r < ii.w; ++r) red_release_gpu(&ydone[ii.z + r], 1u);
            }
          }
          __threadfence_block();
          s_pub = pub + n;  // the producer frees ring slots and activation regions
        }
        __syncwarp();
        pub += n;
        progressed = true;
      }
      // ---- queued activation loads, in order ----
      while (ph < lane0_int(s_pend_tail)) {
        __threadfence_block();  // the entry is read after the count
        const int4 pe = pend[ph % kItemRing];  // (ord, sg, byte offset, phase B | parity << 1)
        const int sg = pe.y, nt = seg_nt[pe.y], p0 = seg_pos[pe.y];
        const bool pb = (pe.w & 1) != 0;
        if (pb) {
          if (!lane0(ld_acquire_gpu(&hdone[sg]) >= (unsigned)bpe_a)) break;
        } else if (!x_ready) {
          if (!lane0(ld_acquire_gpu(xdone) >= gridDim.x)) break;
          x_ready = true;
        }
        if (lane == 0) {
          uint64_t* bar = &act_full[pe.x % kItemRing];
          unsigned char* dst = smem + L.act + pe.z;
          fence_proxy_async_all();  // rows other CTAs wrote, read by the bulk copy
          if (pb) {
            const unsigned size = (unsigned)nt * stride_b;
            mbar_arrive_expect_tx(bar, size);
            bulk_g2s(dst, a.hq + (size_t)p0 * stride_b, size, bar);
          } else {
            mbar_arrive_expect_tx(bar, (unsigned)nt * stride_a);
            for (int t = 0; t < nt; ++t)
              bulk_g2s(dst + (size_t)t * stride_a,
                       a.xg + (size_t)(plist[p0 + t] / a.k) * stride_a, stride_a, bar);
          }
          __threadfence_block();
          s_pend_head = ph + 1;
        }
        __syncwarp();
        ++ph;
        progressed = true;
      }
      // ---- done, or wait (bounded without progress) ----
      if (lane0(s_prod_done != 0) && pub == lane0_int(s_nrec) && ph == lane0_int(s_pend_tail))
        break;
      if (progressed) {
        t_prog = globaltimer();
      } else {
        if (lane0(s_abort != 0)) break;
        if (lane0(globaltimer() - t_prog > kWaitLimitNs)) {
          if (lane == 0) {
            set_error(kErrTimeout);
            s_abort = 1;
          }
          break;
        }
        __nanosleep(64);
      }
    }
  } else if (warp == kWarps) {
    // =============================== producer warp ===============================
    // Takes items, places their activation rows in a circular byte ring (queueing
    // the load for the helper warp) and issues their weight blocks into the stage
    // ring.  Every condition is lane 0's (uniform control flow).
    auto timed_out = [&](unsigned long long t0) -> bool {
      if (lane0(s_abort != 0)) return true;
      if (lane0(globaltimer() - t0 > kWaitLimitNs)) {
        if (lane == 0) {
          set_error(kErrTimeout);
          s_abort = 1;
        }
        return true;
      }
      return false;
    };
    // An item's rows occupy a region [start, start + size) of virtual positions of the
    // ring until the last item using them is published.  Regions are freed in order.
    const unsigned long long ring = 2ull * G.act_buf;
    unsigned long long head = 0, tail = 0;
    int reg_front = 0, reg_cnt = 0;
    auto free_regions = [&]() {
      const int pub = lane0_int(s_pub);
      while (reg_cnt > 0 && reg_last[reg_front] < pub) {
        reg_front = (reg_front + 1) % kItemRing;
        --reg_cnt;
        tail = reg_cnt > 0 ? reg_start[reg_front] : head;
      }
    };
    bool ok = true;
    int gi = 0;                     // blocks issued into the ring
    int cur_key = -1;               // activation set of the newest region
    int cur_tok[kNT] = {-1, -1, -1, -1};
    unsigned cur_off = 0;           // its byte offset in the ring
    unsigned long long cur_start = 0;  // and its virtual position
    unsigned act_par = 0;           // per item ring slot: parity of its next load's phase
    int pend_tail = 0;              // loads queued
    int n_a_items = 0;              // phase-A items taken
    unsigned q0 = 0, q1 = 0;        // items taken ahead (two atomics in flight)
    if (lane == 0) {
      q0 = atomicAdd(work_ctr, 1u);
      q1 = atomicAdd(work_ctr, 1u);
    }
    for (int ord = 0; ok; ++ord) {
      const int item = (int)__shfl_sync(kFull, q0, 0);
      if (item >= n_items) break;
      if (lane == 0) {
        q0 = q1;
        q1 = atomicAdd(work_ctr, 1u);
      }
      const bool phase_b = item >= n_items_a;
      int sg, blk0, nblk;
      if (!phase_b) {
        sg = item / ipa;
        blk0 = (item % ipa) * kBlocksPerItemA;
        nblk = kBlocksPerItemA;
      } else {
        const int j = item - n_items_a;
        if (j < n_items_b2) {
          sg = j / ipb;
          blk0 = (j % ipb) * kBlocksPerItemB;
          nblk = min(kBlocksPerItemB, bpe_b - blk0);
        } else {
          sg = seg_fine + (j - n_items_b2) / bpe_b;
          blk0 = (j - n_items_b2) % bpe_b;
          nblk = 1;
        }
      }
      const int nt = seg_nt[sg], p0 = seg_pos[sg];
      // ---- its ring slot for publication must be free ----
      {
        const unsigned long long t0 = globaltimer();
        while (ok && lane0_int(s_pub) <= ord - kItemRing) {
          if (timed_out(t0)) ok = false;
          __nanosleep(64);
        }
      }
      if (!ok) break;
      // ---- the item's activation rows: the newest region again, or a new one ----
      bool same = false;
      if (!phase_b) {
        same = cur_key == -2;
        for (int t = 0; t < kNT; ++t)
          same = same && cur_tok[t] == (t < nt ? plist[p0 + t] / a.k : -1);
      } else {
        same = cur_key == sg;
      }
      bool act_wait = false, load_par = false;
      free_regions();
      if (same) {  // extend the newest region's life (it may already have been freed)
        if (lane == 0) {
          const int r = (reg_front + reg_cnt + (reg_cnt == 0 ? 0 : -1) + kItemRing) % kItemRing;
          if (reg_cnt == 0) reg_start[r] = cur_start;
          reg_last[r] = ord;
        }
        __syncwarp();
        if (reg_cnt == 0) {
          tail = cur_start;
          reg_cnt = 1;
        }
      } else {
        const unsigned size = (unsigned)nt * (phase_b ? stride_b : stride_a);
        unsigned long long start = 0;
        {
          const unsigned long long t0 = globaltimer();
          for (;;) {
            start = head;
            if (start % ring + size > ring) start = (start / ring + 1) * ring;  // no wrap
            if (start + size - tail <= ring && reg_cnt < kItemRing &&
                pend_tail - lane0_int(s_pend_head) < kItemRing)
              break;
            if (timed_out(t0)) {
              ok = false;
              break;
            }
            __nanosleep(64);
            free_regions();
          }
        }
        if (!ok) break;
        cur_off = (unsigned)(start % ring);
        cur_start = start;
        load_par = (act_par >> (ord % kItemRing)) & 1u;
        act_par ^= 1u << (ord % kItemRing);
        if (lane == 0) {
          const int r = (reg_front + reg_cnt) % kItemRing;
          reg_start[r] = start;
          reg_last[r] = ord;
          pend[pend_tail % kItemRing] =
              make_int4(ord, sg, (int)cur_off, (phase_b ? 1 : 0) | (load_par ? 2 : 0));
          __threadfence_block();
          s_pend_tail = pend_tail + 1;  // the helper warp issues the load
        }
        __syncwarp();
        ++pend_tail;
        if (reg_cnt == 0) tail = start;
        ++reg_cnt;
        head = start + size;
        act_wait = true;
        cur_key = phase_b ? sg : -2;
        for (int t = 0; t < kNT; ++t) cur_tok[t] = (!phase_b && t < nt) ? plist[p0 + t] / a.k : -1;
      }
      // ---- the item's record for publication ----
      if (lane == 0) {
        item_info[ord % kItemRing] = make_int4(phase_b ? 1 : 0, sg, blk0, nblk);
        __threadfence_block();
        s_nrec = ord + 1;
      }
      __syncwarp();
      const int a_ord = phase_b ? 0 : n_a_items++;
      // ---- its blocks into the ring ----
      for (int j = 0; j < nblk && ok; ++j, ++gi) {
        const int st = gi % NS;
        if (gi >= NS) {
          const unsigned long long t0 = globaltimer();
          while (!lane0(mbar_test(&empty[st], ((gi / NS) - 1) & 1))) {
            if (timed_out(t0)) {
              ok = false;
              break;
            }
          }
        }
        if (!ok) break;
        if (lane == 0) {
          const int blk = blk0 + j;
          const int row0 = phase_b ? blk * G.rows_b : blk * kRowsA;
          const int flags = (phase_b ? kSlotPhaseB : 0) | (j == nblk - 1 ? kSlotItemEnd : 0) |
                            (j == 0 && act_wait ? kSlotActWait : 0) |
                            (load_par ? kSlotActPar : 0) |
                            (int)((cur_off >> 7) << kSlotActShift);
          slot_info[st] = make_int4(flags, sg, row0, ord | (a_ord << 16));
          unsigned char* buf = smem + L.stages + (size_t)st * G.stage_bytes;
          fence_proxy_async();
          if (!phase_b) {
            const size_t r0 = (size_t)uniq[seg_slot[sg]] * a.I + row0;
            const size_t qrow = a.H / 8, srow = a.H / 64;
            mbar_arrive_expect_tx(&full[st], G.a_bytes);
            bulk_g2s(buf, a.gq + r0 * qrow, G.a_q, &full[st]);
            bulk_g2s(buf + G.a_q, a.gs + r0 * srow, G.a_sb, &full[st]);
            if (F != kFmtMx) bulk_g2s(buf + G.a_q + G.a_sb, a.gb + r0 * srow, G.a_sb, &full[st]);
            buf += G.a_mat;
            bulk_g2s(buf, a.uq + r0 * qrow, G.a_q, &full[st]);
            bulk_g2s(buf + G.a_q, a.us + r0 * srow, G.a_sb, &full[st]);
            if (F != kFmtMx) bulk_g2s(buf + G.a_q + G.a_sb, a.ub + r0 * srow, G.a_sb, &full[st]);
          } else {
            const int nrows = min(G.rows_b, a.H - row0);
            const size_t r0 = (size_t)uniq[seg_slot[sg]] * a.H + row0;
            const size_t qrow = a.I / 8, srow = a.I / 64;
            const unsigned qb = nrows * (a.I / 2), sb = nrows * (a.I / 32);
            mbar_arrive_expect_tx(&full[st], qb + (F == kFmtMx ? 1 : 2) * sb);
            bulk_g2s(buf, a.dq + r0 * qrow, qb, &full[st]);
            bulk_g2s(buf + G.b_q, a.ds + r0 * srow, sb, &full[st]);
            if (F != kFmtMx) bulk_g2s(buf + G.b_q + G.b_sb, a.db + r0 * srow, sb, &full[st]);
          }
        }
        __syncwarp();
      }
    }
    // ---- the end marker ----
    if (ok) {
      const int st = gi % NS;
      if (gi >= NS) {
        const unsigned long long t0 = globaltimer();
        while (!lane0(mbar_test(&empty[st], ((gi / NS) - 1) & 1))) {
          if (timed_out(t0)) {
            ok = false;
            break;
          }
        }
      }
      if (ok && lane == 0) {
        slot_info[st] = make_int4(kSlotEnd, 0, 0, 0);
        mbar_arrive(&full[st]);
      }
      __syncwarp();
    }
    if (lane == 0) {
      __threadfence_block();
      s_prod_done = 1;
    }
    // copies still in flight after an abort land before the CTA exits (bounded)
    if (!ok && lane == 0) {
      for (int g = (gi > NS ? gi - NS : 0); g < gi; ++g) {
        const unsigned long long t0 = globaltimer();
        while (!mbar_test(&full[g % NS], (g / NS) & 1) && globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
    __syncwarp();
  } else {
    // ================================ compute warps ================================
    uint16_t* hscr = reinterpret_cast<uint16_t*>(smem + L.hscr);  // [kItemRing][kNT][32]
    auto wait_cons = [&](uint64_t* bar, unsigned parity) -> bool {
      if (s_abort) return false;
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(bar, parity)) {
        if (s_abort) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
          set_error(kErrTimeout);
          s_abort = 1;
          return false;
        }
      }
      return true;
    };
    for (int gi = 0;; ++gi) {
      const int st = gi % NS;
      if (!wait_cons(&full[st], (gi / NS) & 1)) break;
      const int4 si = slot_info[st];
      if (si.x & kSlotEnd) break;
      const bool phase_b = (si.x & kSlotPhaseB) != 0;
      const int sg = si.y, row0 = si.z, ord = si.w & 0xffff, a_ord = si.w >> 16;
      if ((si.x & kSlotActWait) &&
          !wait_cons(&act_full[ord % kItemRing], (si.x & kSlotActPar) ? 1u : 0u))
        break;
      const int nt = seg_nt[sg], p0 = seg_pos[sg];
      const unsigned char* act = smem + L.act + ((size_t)(si.x >> kSlotActShift) << 7);
      const unsigned char* buf = smem + L.stages + (size_t)st * G.stage_bytes;
      float Gs[kNT], Us[kNT];
      float v = 0.f;
      int vid = -1, nrows = 0;
      if (!phase_b) {
        const unsigned char* bgq = buf + (size_t)warp * (a.H / 2);
        const uint16_t* bgs = reinterpret_cast<const uint16_t*>(buf + G.a_q) + warp * (a.H / 64);
        const uint16_t* bgb = reinterpret_cast<const uint16_t*>(buf + G.a_q + G.a_sb) + warp * (a.H / 64);
        const unsigned char* bu = buf + G.a_mat;
        const unsigned char* buq = bu + (size_t)warp * (a.H / 2);
        const uint16_t* bus = reinterpret_cast<const uint16_t*>(bu + G.a_q) + warp * (a.H / 64);
        const uint16_t* bub = reinterpret_cast<const uint16_t*>(bu + G.a_q + G.a_sb) + warp * (a.H / 64);
        switch (nt) {
          case 1: dispatch_a<1, F>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, act, stride_a, lane, Gs, Us); break;
          case 2: dispatch_a<2, F>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, act, stride_a, lane, Gs, Us); break;
          case 3: dispatch_a<3, F>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, act, stride_a, lane, Gs, Us); break;
          default: dispatch_a<4, F>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, act, stride_a, lane, Gs, Us); break;
        }
      } else {
        nrows = min(G.rows_b, a.H - row0);
        const uint16_t* bs = reinterpret_cast<const uint16_t*>(buf + G.b_q);
        const uint16_t* bb = reinterpret_cast<const uint16_t*>(buf + G.b_q + G.b_sb);
        switch (nt) {
          case 1: v = dispatch_b<1, F>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, act, stride_b, lane, vid); break;
          case 2: v = dispatch_b<2, F>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, act, stride_b, lane, vid); break;
          case 3: v = dispatch_b<3, F>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, act, stride_b, lane, vid); break;
          default: v = dispatch_b<4, F>(G.rounds_b, buf, bs, bb, warp, nrows, a.I, act, stride_b, lane, vid); break;
        }
      }
      // this warp is done reading stage st
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      const bool item_end = (si.x & kSlotItemEnd) != 0;
      if (!phase_b) {
        uint16_t* hs = hscr + (ord % kItemRing) * (kNT * 32);
        if (lane < nt) {
          float gv = 0.f, uv = 0.f;
#pragma unroll
          for (int t = 0; t < kNT; ++t)
            if (t == lane) {
              gv = Gs[t];
              uv = Us[t];
            }
          const float g = round_to_bf16(gv), hu = round_to_bf16(uv);
          // silu(g) = g / (1 + e^-g); the fast division's error (2 ulp of fp32) is far
          // below the bf16 step h is rounded to
          const uint16_t hb = float_to_bf16_bits(__fdividef(g, 1.0f + __expf(-g)) * hu);
          a.h[(size_t)(p0 + lane) * a.I + row0 + warp] = hb;
          hs[lane * 32 + (row0 & 31) + warp] = hb;
        }
        // (the item's 32 h rows per pair form one chunk of h; the producer converts it
        // to the fixed-point layout when it publishes the item)
      } else if (vid >= 0) {
        const int r = warp + kWarps * (vid / kNT), t = vid % kNT;
        if (r < nrows) a.y[(size_t)(p0 + t) * a.H + row0 + r] = v;
      }
      if (item_end) {  // this warp's stores of the item are done (released at CTA scope)
        __syncwarp();
        if (lane == 0) mbar_arrive(&item_done[ord % kItemRing]);
      }
    }
  }

  // ---- combine: row blocks blockIdx.x, blockIdx.x + grid, ... once complete ----
  // out[t][c] = bf16(sum_j w[t,j] * y[pos(t,j)][c]): a group of gk lanes (gk = k
  // rounded up to a power of two, at most 32) per output, lane j of the group
  // taking pairs j, j+gk, ...; the group sums in a fixed shuffle order.
  __syncthreads();
  {
    const int n_rb = (a.H + G.rows_b - 1) / G.rows_b;
    int gk = 1;
    while (gk < a.k && gk < 32) gk <<= 1;
    const int gl = lane & (gk - 1);
    const int per_rb = a.T * G.rows_b;
    const int groups = kThreads / gk;
    for (int rb = blockIdx.x; rb < n_rb; rb += gridDim.x) {
      if (threadIdx.x == 0) {
        const unsigned long long t0 = globaltimer();
        while (!s_abort && ld_acquire_gpu(&ydone[rb]) < (unsigned)nseg) {
          if (globaltimer() - t0 > kWaitLimitNs) {
            set_error(kErrTimeout);
            s_abort = 1;
          }
        }
        __threadfence();
      }
      __syncthreads();
      for (int o0 = 0; o0 < per_rb; o0 += groups) {  // uniform trip count: every lane shuffles
        const int o = o0 + (int)threadIdx.x / gk;
        const int t = o / G.rows_b, c = rb * G.rows_b + o % G.rows_b;
        const bool valid = o < per_rb && c < a.H;
        float acc = 0.f;
        if (valid)
          for (int j = gl; j < a.k; j += gk) {
            const int p = t * a.k + j;
            const int pos = pos_of[p];
            if (pos >= 0) acc = fmaf(__ldg(a.w + p), __ldcg(a.y + (size_t)pos * a.H + c), acc);
          }
        for (int m = gk >> 1; m >= 1; m >>= 1) acc += __shfl_xor_sync(kFull, acc, m);
        if (valid && gl == 0) a.out[(size_t)t * a.H + c] = float_to_bf16_bits(acc);
      }
      if (threadIdx.x == 0) ydone[rb] = 0;  // for the next call
    }
  }
  grid_dep_launch();
  // ---- the CTA that finishes last resets the other counters ----
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(exit_cnt, 1u);
    if (old == gridDim.x - 1) {
      for (int sgi = 0; sgi < nseg; ++sgi) hdone[sgi] = 0;
      *work_ctr = 0;
      *xdone = 0;
      *exit_cnt = 0;
      __threadfence();
    }
  }
}

}  // namespace qeg
