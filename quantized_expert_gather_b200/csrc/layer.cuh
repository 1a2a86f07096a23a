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
//             to `seg` of its pairs.  A window whose x rows fit one activation
//             buffer keeps them all in shared memory (converted while the union
//             forms);
//   phase A   gate+up over blocks of 8 rows (segment, rows of Wg and Wu):
//               h = bf16(silu(bf16(Wg x)) * bf16(Wu x))
//             (the one-pass epilogue of "Apple7/8 MoE gate and up in one decode
//             pass", splash PR 45, "What changed"), h written to the workspace;
//   phase B   down over blocks of rows_b rows of Wd: y = Wd h per pair, fp32.
//             A segment's phase-B blocks start once every phase-A block of that
//             segment has published (counter hdone[seg]);
//   combine   out[t] = bf16(sum_j w[t,j] * y[t,j]) per block of rows_b output
//             rows, by CTA (row block mod grid) once every segment of the row
//             block has published (counter ydone[rb]).
// Each CTA takes a contiguous share of all phase-A blocks (segment order), then
// of all phase-B blocks, balanced by cost (a block's bytes are the same for every
// segment; its compute grows with the segment's pairs), so the CTAs finish
// together, and a CTA's share spans few segments, so its activation sets change
// rarely.  An
// expert with more than `seg` pairs in the window forms several segments and is
// streamed once per segment.  Every spin on a counter or barrier is bounded
// (common.cuh); the counters are zero again when the kernel ends.
//
// Warps: 16 compute warps in two teams of 8, one producer warp and one helper
// warp.  The producer issues this CTA's weight blocks into a ring of stages (1-D
// bulk copies, mbarrier completion); the helper publishes finished blocks to the
// other CTAs (counter release reductions); the teams take alternate blocks, and
// all compute warps convert each new activation set (the segment's x rows for
// phase A, its h rows for phase B) into shared memory together.
//
// Compute: each warp owns whole rows of its team's block (phase A: one row of Wg
// and the same row of Wu; phase B: up to 4 rows of Wd) over the full input width,
// one pair at a time.  Lane l takes
// the 32-column chunks l, l+32, ... of its rows, so one lane chunk sits inside
// one quantisation group (64 columns affine, 32 mxfp4):
//     partial = s * sum_c q_c x_c + b * sum_c x_c.
// Activations are 16-bit block fixed point (one exponent per 32-column chunk,
// see below), so that sum_c q_c x_c is an exact integer dot product of the 4-bit
// codes with the activation's two bytes (dp4a), scaled once per chunk.  A warp
// reduces its rows over its lanes once per block.
#pragma once

#include "common.cuh"
#include "router.cuh"
#include "union.cuh"

namespace qeg {

// Bank formats.  kFmtAffine: 4-bit codes, bf16 scale and bias per 64 columns
// (w = s q + b).  kFmtMx: mxfp4, e2m1 codes and one e8m0 scale per 32 columns
// (w = e2m1(q) 2^(e - 127)).  Codes are packed alike in both.
constexpr int kFmtAffine = 0;
constexpr int kFmtMx = 1;

constexpr int kTeamWarps = 8;                // compute warps per team (rows per block)
constexpr int kTeams = 2;                    // teams, taking alternate blocks
constexpr int kWarps = kTeams * kTeamWarps;  // compute warps
constexpr int kConsumerThreads = 32 * kWarps;
constexpr int kThreads = kConsumerThreads + 64;  // + a producer warp and a helper warp
constexpr int kRowsA = kTeamWarps;  // phase A: one row of gate and of up per warp per block
constexpr int kMaxRowsPerWarpB = 4; // phase B: rows of Wd per warp per block
// Ring depth: 4, or 2 when shared memory is short.  Always even: block j sits in
// stage j % depth and belongs to team j % 2, so with an even depth every stage is
// used by one team only, and a team's parity wait on a stage can never be more than
// one phase ahead of that stage (an odd depth would let one team's wait for a later
// block pass on the phase of the other team's block still in flight; waiting first
// for the stage's previous block to be consumed avoids that, but couples the teams
// and measured slower with 5 stages than with 4).
constexpr int kMaxStages = 4;
constexpr int kNT = 2;              // pairs per compute pass (phase A; phase B takes one)
constexpr int kMaxPairsFused = 1024;
constexpr unsigned kBarUnion = 1;   // named barrier: union formed (warp 0 -> producer)
constexpr unsigned kBarWork = 2;    // named barrier: every warp but the producer
constexpr int kRouteWarps = kWarps;  // warps picking the experts when the router is fused
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
  int rows_b;              // phase B rows per block (multiple of kTeamWarps, <= 32)
  unsigned a_q, a_sb, a_mat, a_bytes;  // phase A block: per matrix codes / scale (or bias) bytes
  unsigned b_q, b_sb, b_bytes;         // phase B full block
  unsigned stage_bytes;
  // shared-memory plan (layer_plan): index tables at offset 0, then the stage ring,
  // then the activation area.  Normal layout: `stages` stages and act_n bytes; wide
  // layout (windows where one expert has more pairs than act_n holds rows of x):
  // stages_w stages and act_w bytes, every x row of the window resident (0: none)
  unsigned tables;
  int stages, stages_w;
  unsigned act_n, act_w;
  unsigned total;          // dynamic shared memory of the launch
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
  int rb = (16 * H / I) / kTeamWarps * kTeamWarps;  // about one phase-A stage of Wd rows
  if (rb < kTeamWarps) rb = kTeamWarps;
  if (rb > kTeamWarps * kMaxRowsPerWarpB) rb = kTeamWarps * kMaxRowsPerWarpB;
  g.rows_b = rb;
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
  g.tables = 0;
  g.stages = g.stages_w = 0;
  g.act_n = 0;
  g.act_w = 0;
  g.total = 0;
  return g;
}

// Index tables at the start of shared memory: union scratch and result, the pair
// maps, and the segment tables of phase A and of phase B (at most P each).
struct LayerSmem {
  size_t cnt, rank, unique, offsets, pair_list, pos_of, tok_of, sa_slot, sa_pos, sa_nt, sb_slot,
      sb_pos, sb_nt, ridx, rw, end;
};
// `routed`: the kernel picks the experts itself from router logits, and the picks and
// their weights (P ints, P floats) are kept here too.
__host__ __device__ inline LayerSmem layer_smem(int E, int P, bool routed = false) {
  LayerSmem s;
  const int m = (E < P ? E : P) > 0 ? (E < P ? E : P) : 1;
  s.cnt = 0;
  s.rank = align_up(s.cnt + sizeof(int) * E, 16);
  s.unique = align_up(s.rank + sizeof(int) * P, 16);
  s.offsets = align_up(s.unique + sizeof(int) * m, 16);
  s.pair_list = align_up(s.offsets + sizeof(int) * (m + 1), 16);
  s.pos_of = align_up(s.pair_list + sizeof(int) * P, 16);
  s.tok_of = align_up(s.pos_of + sizeof(int) * P, 16);
  s.sa_slot = align_up(s.tok_of + sizeof(int) * P, 16);
  s.sa_pos = align_up(s.sa_slot + sizeof(int) * P, 16);
  s.sa_nt = align_up(s.sa_pos + sizeof(int) * P, 16);
  s.sb_slot = align_up(s.sa_nt + sizeof(int) * P, 16);
  s.sb_pos = align_up(s.sb_slot + sizeof(int) * P, 16);
  s.sb_nt = align_up(s.sb_pos + sizeof(int) * P, 16);
  s.ridx = align_up(s.sb_nt + sizeof(int) * P, 16);
  s.rw = align_up(s.ridx + (routed ? sizeof(int) * P : 0), 16);
  s.end = align_up(s.rw + (routed ? sizeof(float) * P : 0), 128);
  return s;
}

// The shared-memory plan for a window of T tokens, top-k, within `budget` bytes: the
// deepest normal ring (kMaxStages or 2 stages) that leaves at least two x rows and
// min(T, 8) h rows of activations, the rest of the budget being the activation area; and a wide
// layout holding all T x rows when that needs more than the normal area (its ring at
// least 2 stages deep and even, else none).  False if not even the normal layout fits.
__host__ __device__ inline bool layer_plan(LayerGeom& g, int E, int T, int k, size_t budget,
                                           bool routed = false) {
  const int P = T * k;
  g.tables = (unsigned)layer_smem(E, P, routed).end;
  const size_t ra = act_bytes(g.rounds_a), rbb = act_bytes(g.rounds_b);
  // an expert has at most T pairs in the window, so min(T, 8) h rows hold its set
  const size_t hmin = (size_t)(T < 8 ? T : 8) * rbb;
  const size_t act_min = align_up(2 * ra > hmin ? 2 * ra : hmin, 128);
  g.stages = 0;
  for (int st = kMaxStages; st >= 2; st -= 2) {
    const size_t used = (size_t)g.tables + (size_t)st * g.stage_bytes;
    if (used + act_min <= budget) {
      g.stages = st;
      g.act_n = (unsigned)((budget - used) / 128 * 128);
      break;
    }
  }
  if (g.stages == 0) return false;
  g.stages_w = 0;
  g.act_w = (unsigned)align_up((size_t)T * ra, 128);
  if (g.act_w > g.act_n) {
    const size_t room = budget > (size_t)g.tables + g.act_w ? budget - g.tables - g.act_w : 0;
    int st = (int)(room / g.stage_bytes);
    if (st > kMaxStages) st = kMaxStages;
    st &= ~1;  // even (see kMaxStages)
    if (st >= 2) g.stages_w = st;
  }
  g.total = (unsigned)budget;
  return true;
}

// Workspace counters (unsigned), a region of fixed size at the start of every
// workspace so that calls of different shapes never see each other's data there:
// [0] CTAs finished, [1, 1+kMaxPairsFused) hdone per distinct expert (phase-A
// blocks published), then ydone per phase-B row block (at most kMaxRowBlocks),
// then two words kept zero.
constexpr int kMaxRowBlocks = 4096 / kTeamWarps;
constexpr size_t kSyncWords = 1 + kMaxPairsFused + kMaxRowBlocks + 2;

// -------------------------------------------------------------- arguments ---
struct LayerArgs {
  const uint16_t* x;  // [T, H] bf16
  const int* idx;     // [T, k]
  const float* w;     // [T, k]
  const uint32_t *gq, *uq, *dq;
  const uint16_t *gs, *gb, *us, *ub, *ds, *db;
  uint16_t* h;        // workspace [P, I] bf16, rows in pair_list order
  float* y;           // workspace [P, H] fp32, rows in pair_list order
  unsigned* sync;     // workspace counters (kSyncWords)
  int *ex_u, *ex_unique, *ex_offsets, *ex_pair_list;  // union export (CTA 0), may be null
  uint16_t* out;      // [T, H] bf16
  int T, k, E, H, I;
  LayerGeom g;
  int wait_prior;     // wait for the preceding grid before reading any input
  int x_res;          // every x row of the window fits one activation buffer: each CTA
                      // keeps them all in shared memory for phase A
  // Router step fused ahead of the union (idx and w unused): [T, E] fp32 logits, top-k
  // of their softmax per token, renormalised over the k when renorm is set; CTA 0
  // writes the picks and weights to ridx_out / rw_out ([T, k]).
  const float* logits;
  int renorm;
  int* ridx_out;
  float* rw_out;
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
// integers by dp4a over 4-bit codes: the affine codes of a 32-bit word w are split
// into qa = w & 0x0F0F0F0F (columns 0, 2, 4, 6 of the word, one per byte) and
// qb = w & 0xF0F0F0F0 (columns 1, 3, 5, 7, each as 16 q); mxfp4 codes become bytes
// by table lookup in column order 0..3 and 4..7 (split_codes_mx).
//
// Layout of one activation row (a token's x or a pair's h) of D columns, R rounds
// (R >= D / 1024), in act_bytes(R) = 2304 R bytes: for chunk ch = i * 32 + l
// (i < R, l < 32) the uint4 at index (i * 4 + m) * 32 + l covers columns
// 32 ch + 8m .. +7 as (affine)
//   .x = low bytes of columns 8m+0,2,4,6   .y = low bytes of 8m+1,3,5,7
//   .z = high bytes of columns 8m+0,2,4,6  .w = high bytes of 8m+1,3,5,7
// or (mxfp4) .x / .z = low / high bytes of columns 8m+0..3, .y / .w of 8m+4..7,
// followed (at byte 2048 R) by float2 sc[ch] = (2^(e - 14) (2^(e - 18) in the affine
// layout, whose chunk sums are 16 times too large), sum of the chunk's 32
// values).  Resident x rows and every activation set use it, in shared memory.
constexpr uint32_t kNibbleBytes = 0x0F0F0F0Fu;

__device__ __forceinline__ int dp4a_lo(uint32_t q, uint32_t d, int c) {
  return static_cast<int>(__dp4a(q, d, static_cast<unsigned>(c)));
}
__device__ __forceinline__ int dp4a_hi(uint32_t q, uint32_t d, int c) {
  int r;  // unsigned code bytes times signed activation bytes
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(r) : "r"(q), "r"(d), "r"(c));
  return r;
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
// partial sums keep the dp4a dependency chains short.  In the affine format the
// odd codes stay in the high nibble of their byte (16 q, see split_codes), so the
// affine result is 16 * sum q v (|.| < 2^28; the chunk scale carries the 1/16).
template <int F>
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
  if constexpr (F == kFmtMx) return (hi0 + hi1) * 256 + (lo0 + lo1);
  else return (((hi0 << 4) + hi1) << 8) + ((lo0 << 4) + lo1);
}

// The 32 codes of a uint4, split as described above (affine format), except that
// the odd codes are left in the high nibble of their byte: qs[2m+1] = w & 0xF0F0F0F0
// holds 16 q per byte (one operation less per word; chunk_dot accounts for it).
__device__ __forceinline__ void split_codes(const uint4 v, uint32_t (&qs)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    qs[2 * m] = w[m] & kNibbleBytes;
    qs[2 * m + 1] = w[m] & ~kNibbleBytes;
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
    // (chunk_dot returns 16 x the sum in this format; the activation scale holds 1/16)
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
  // affine chunk sums come out 16 times too large (chunk_dot): the row's scale
  // carries the 1/16 (exact, a power of two)
  if (F != kFmtMx) scale *= 0.0625f;
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

__device__ __forceinline__ void red_relaxed_gpu(unsigned* p, unsigned v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Spin (bounded) until *p >= target.  Returns false and sets kErrTimeout if the
// limit runs out.
__device__ __forceinline__ bool wait_counter(const unsigned* p, unsigned target) {
  if (ld_acquire_gpu(p) >= target) return true;
  const unsigned long long t0 = globaltimer();
  while (ld_acquire_gpu(p) < target) {
    __nanosleep(32);
    if (globaltimer() - t0 > wait_limit()) {
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
                                       const unsigned char* const (&act)[kNT], int lane,
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
        const unsigned char* row = act[t];
        uint4 xd[4];
        load_xq(row, i, lane, xd);
        const float2 sc = load_sc(row, R, ch);
        const float dg = static_cast<float>(chunk_dot<F>(qg, xd));
        const float du = static_cast<float>(chunk_dot<F>(qu, xd));
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

// Phase B: rows row0 + kTeamWarps*q (q < kMaxRowsPerWarpB, rows < nrows) of Wd, NT pairs.
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
        const int r = row0 + kTeamWarps * q;
        if (r < nrows) {
          uint32_t qs[8];
          split_codes_f<F>(*reinterpret_cast<const uint4*>(bq + (size_t)r * qstride + ch * 16), qs);
          // a row's scales: I/64 bf16 (affine) or I/32 bytes (mxfp4), I/32 bytes either way
          const float2 sb = chunk_sb<F>(bs + r * sstride, bb + r * sstride, ch);
          const float sv = sb.x, bv = sb.y;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float d = static_cast<float>(chunk_dot<F>(qs, xd[t]));
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
                                           const unsigned char* const (&act)[kNT], int lane,
                                           float (&G)[kNT], float (&U)[kNT]) {
  if (R == 1) rows_a<NT, 1, F>(bgq, bgs, bgb, buq, bus, bub, H, act, lane, G, U);
  else if (R == 2) rows_a<NT, 2, F>(bgq, bgs, bgb, buq, bus, bub, H, act, lane, G, U);
  else if (R == 4) rows_a<NT, 4, F>(bgq, bgs, bgb, buq, bus, bub, H, act, lane, G, U);
  else if (R == 6) rows_a<NT, 6, F>(bgq, bgs, bgb, buq, bus, bub, H, act, lane, G, U);
  else rows_a<NT, 8, F>(bgq, bgs, bgb, buq, bus, bub, H, act, lane, G, U);
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

constexpr int kPubRing = 16;      // blocks between compute and publication

// Activation set (the rows of one segment's pairs) into `buf`, by the compute warps
// (kConsumerThreads threads): phase A converts the pairs' token rows of x, phase B the pairs' rows
// of h (written by other CTAs; read around L1).  Four consecutive lanes convert one
// 32-column chunk together.
template <int F>
__device__ __forceinline__ void convert_set(const LayerArgs& a, const LayerGeom& G, bool phase_b,
                                            const int* tok_of, int p0, int nt,
                                            unsigned char* buf, int lane, int tid = threadIdx.x,
                                            int nthreads = kConsumerThreads) {
  const int D = phase_b ? a.I : a.H, R = phase_b ? G.rounds_b : G.rounds_a, nch = D / 32;
  const unsigned stride = act_bytes(R);
  const int nq = nt * nch * 4;  // quarters of 8 columns
  // kBatch quarters per thread at a time: their loads are all issued before the first
  // conversion waits on one
  constexpr int kBatch = 4;
  for (int q0 = tid; q0 < nq; q0 += kBatch * nthreads) {
    uint4 v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int q = q0 + i * nthreads;
      v[i] = make_uint4(0u, 0u, 0u, 0u);
      if (q < nq) {
        const int m = q & 3, tc = q >> 2, t = tc / nch, ch = tc % nch;
        if (phase_b)
          v[i] = __ldcg(reinterpret_cast<const uint4*>(a.h + (size_t)(p0 + t) * a.I + ch * 32 + m * 8));
        else
          v[i] = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)tok_of[p0 + t] * a.H + ch * 32 +
                                                      m * 8));
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int q = q0 + i * nthreads;
      if (q < nq) {  // the four lanes of a chunk agree (nq is a multiple of 4)
        const int m = q & 3, tc = q >> 2, t = tc / nch, ch = tc % nch;
        uint4 packed;
        const float2 sc = fixed_point_quarter<F>(v[i], 0xfu << (lane & ~3), packed);
        unsigned char* row = buf + (size_t)t * stride;
        reinterpret_cast<uint4*>(row)[((ch / 32) * 4 + m) * 32 + (ch % 32)] = packed;
        if (m == 0) reinterpret_cast<float2*>(row + act_digit_bytes(R))[ch] = sc;
      }
    }
  }
}

// Rows of x resident in shared memory: all T tokens, by the threads [t0, t0 + nthr)
// of this CTA (four consecutive lanes per 32-column chunk).
template <int F>
__device__ __forceinline__ void convert_x_all(const LayerArgs& a, const LayerGeom& G,
                                              unsigned char* xres, int t0, int nthr, int lane) {
  const int nch = a.H / 32, R = G.rounds_a;
  const unsigned stride = act_bytes(R);
  const int nq = a.T * nch * 4;  // quarters of 8 columns
  constexpr int kBatch = 4;      // loads issued before the first conversion
  for (int q0 = t0; q0 < nq; q0 += kBatch * nthr) {
    uint4 v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int q = q0 + i * nthr;
      v[i] = make_uint4(0u, 0u, 0u, 0u);
      if (q < nq) {
        const int m = q & 3, tc = q >> 2, t = tc / nch, ch = tc % nch;
        v[i] = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H + ch * 32 + m * 8));
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int q = q0 + i * nthr;
      if (q < nq) {  // the four lanes of a chunk agree (nq and nthr are multiples of 4)
        const int m = q & 3, tc = q >> 2, t = tc / nch, ch = tc % nch;
        uint4 packed;
        const float2 sc = fixed_point_quarter<F>(v[i], 0xfu << (lane & ~3), packed);
        unsigned char* row = xres + (size_t)t * stride;
        reinterpret_cast<uint4*>(row)[((ch / 32) * 4 + m) * 32 + (ch % 32)] = packed;
        if (m == 0) reinterpret_cast<float2*>(row + act_digit_bytes(R))[ch] = sc;
      }
    }
  }
}

// Segment table: expert slot i (n_i pairs) contributes ceil(n_i / seg) segments of at
// most `seg` pairs, in slot order.  Run by one warp; returns the number of segments.
__device__ __forceinline__ int make_segments(const int* offs, int u, int seg, int* s_slot,
                                             int* s_pos, int* s_nt, int lane) {
  int base = 0;
  for (int b0 = 0; b0 < u; b0 += 32) {
    const int i = b0 + lane;
    const int n_i = (i < u) ? offs[i + 1] - offs[i] : 0;
    const int c = (n_i + seg - 1) / seg;
    int incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, d);
      if (lane >= d) incl += v;
    }
    for (int j = 0; j < c; ++j) {
      const int sidx = base + incl - c + j;
      s_slot[sidx] = i;
      s_pos[sidx] = offs[i] + j * seg;
      s_nt[sidx] = min(seg, n_i - j * seg);
    }
    base += __shfl_sync(kFull, incl, 31);
  }
  return base;
}

// Cost of one block of a segment of nt pairs, in units of about 10 ns of a team's time
// (fitted to per-block timings on B200 at hidden 4096 / inter 2048): phase A runs its
// pairs two per pass over the block's codes, phase B one per pass.  Only costs within
// one phase are compared with each other.
__device__ __forceinline__ unsigned block_cost(bool phase_b, int nt) {
  return phase_b ? 36u + 119u * (unsigned)nt
                 : 26u + 73u * (unsigned)nt + 64u * (unsigned)((nt + 1) >> 1);
}
// A CTA whose share of a phase-B range crosses a segment start converts one more
// activation set than the others: about 2.5 us for each team, both teams at once, in
// the units of the summed block costs of both teams.  Half of it is charged to the
// segment's first block and half to its last, so that a share that starts or ends at
// a segment start, and converts nothing extra, is charged half.
constexpr unsigned kSetCost = 500u;

// Inclusive prefix of the segments' costs, pref[s] = sum over segments s' <= s of
// bpe block_cost(nt[s']) + sig.  Run by one warp.
__device__ __forceinline__ unsigned prefix_costs(const int* nt, int nseg, int bpe, bool phase_b,
                                                 unsigned sig, unsigned* pref, int lane) {
  unsigned base = 0;
  for (int b0 = 0; b0 < nseg; b0 += 32) {
    const int sidx = b0 + lane;
    const unsigned c = sidx < nseg ? (unsigned)bpe * block_cost(phase_b, nt[sidx]) + sig : 0u;
    unsigned incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const unsigned v = __shfl_up_sync(kFull, incl, d);
      if (lane >= d) incl += v;
    }
    if (sidx < nseg) pref[sidx] = base + incl;
    base += __shfl_sync(kFull, incl, 31);
  }
  return base;
}

// Cost of the blocks before block b (global index, segments in order, bpe blocks each):
// a segment's first block carries sig / 2 more, its last block the rest of sig.  One
// thread.
__device__ __forceinline__ unsigned cost_before(const unsigned* pref, const int* nt, int b, int bpe,
                                                bool phase_b, unsigned sig) {
  const int sg = b / bpe, i = b - sg * bpe;
  const unsigned before = sg > 0 ? pref[sg - 1] : 0u;
  return i == 0 ? before : before + sig / 2u + (unsigned)i * block_cost(phase_b, nt[sg]);
}

// First block (global index) of segments [s0, s1) whose cost_before reaches t: the
// start of a CTA's share.  One thread.
__device__ __forceinline__ int block_at(const unsigned* pref, const int* nt, int s0, int s1,
                                        int bpe, unsigned t, bool phase_b, unsigned sig) {
  const unsigned before0 = s0 > 0 ? pref[s0 - 1] : 0u;
  if (t <= before0) return s0 * bpe;
  if (s1 <= s0 || t > pref[s1 - 1]) return s1 * bpe;
  int lo = s0, hi = s1 - 1;  // first s in [lo, hi] with pref[s] >= t
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (pref[mid] >= t) hi = mid;
    else lo = mid + 1;
  }
  const unsigned before = lo > 0 ? pref[lo - 1] : 0u, w = block_cost(phase_b, nt[lo]);
  const unsigned d = t - before, h = sig / 2u;  // 0 < d <= sig + bpe w
  return lo * bpe + (d <= h + w ? 1 : min(bpe, (int)((d - h + w - 1) / w)));
}

// This CTA's block ranges, r0..r7 (lane q returns rq): phase A group 1 [r0, r1) and
// group 2 [r2, r3), phase B group 1 [r4, r5) and group 2 [r6, r7), each a share of its
// group's blocks, the shares in blockIdx order.  Group 1 is the experts up to the one
// holding the middle of the phase-A cost, group 2 the rest.  A CTA streams its phase-A
// share of group 1, then of group 2, then its phase-B share of group 1, then of group
// 2: by the time it reaches group 1's phase B, every CTA has long finished group 1's
// phase A (nobody waits for h at the turn from A to B), and group 2's phase A finishes
// while the CTAs stream group 1's phase B.
// Each range is cut where its cost prefix reaches a CTA's ideal share, corrected by the
// cost the ranges cut before it gave the CTAs before this one beyond their ideal (the
// rounding error carried from range to range): a CTA's total stays within about a block
// of the mean instead of collecting the rounding of all four ranges.  The correction is
// at most half of a CTA's ideal share of the range, which keeps the cuts in blockIdx
// order.  Lanes 0 and 1 cut at blockIdx and blockIdx + 1.  Run by one warp; prefA /
// prefB are scratch for nsa / nsb unsigned.
__device__ __forceinline__ int plan_shares(const int* sa_slot, const int* sa_nt, int nsa,
                                           int bpe_a, const int* sb_slot, const int* sb_nt,
                                           int nsb, int bpe_b, unsigned* prefA, unsigned* prefB,
                                           int lane) {
  const unsigned totA = prefix_costs(sa_nt, nsa, bpe_a, false, 0u, prefA, lane);
  const unsigned totB = prefix_costs(sb_nt, nsb, bpe_b, true, kSetCost, prefB, lane);
  __syncwarp();
  // group 1: phase-A segments up to the one holding the middle of the cost, and the
  // phase-B segments of the same experts
  int nsa1 = 0;
  for (int b0 = 0; b0 < nsa; b0 += 32) {
    const int sidx = b0 + lane;
    const unsigned hit = __ballot_sync(kFull, sidx < nsa && 2u * prefA[sidx] >= totA);
    if (hit) {
      nsa1 = b0 + __ffs(hit);  // one past the middle segment
      break;
    }
  }
  const int umid = nsa1 > 0 ? sa_slot[nsa1 - 1] + 1 : 0;
  int nsb1 = nsb;
  for (int b0 = 0; b0 < nsb; b0 += 32) {
    const int sidx = b0 + lane;
    const unsigned hit = __ballot_sync(kFull, sidx < nsb && sb_slot[sidx] >= umid);
    if (hit) {
      nsb1 = b0 + __ffs(hit) - 1;
      break;
    }
  }
  int cut[4] = {0, 0, 0, 0};  // range q = 2 phase + group: A1, A2, B1, B2
  if (lane < 2) {
    const unsigned long long k = blockIdx.x + (unsigned)lane, G = gridDim.x;
    long long err = 0;  // cost the ranges cut so far gave CTAs 0 .. k-1 beyond their ideal
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = (i + 2) & 3;  // B1, B2, A1, A2
      const bool pb = q >= 2;
      const int g = q & 1;
      const unsigned* pref = pb ? prefB : prefA;
      const int* nt = pb ? sb_nt : sa_nt;
      const int n1 = pb ? nsb1 : nsa1, n = pb ? nsb : nsa, bpe = pb ? bpe_b : bpe_a;
      const unsigned tot = pb ? totB : totA, sig = pb ? kSetCost : 0u;
      const unsigned c1 = n1 > 0 ? pref[n1 - 1] : 0u;
      const unsigned base = g ? c1 : 0u, cg = g ? tot - c1 : c1;
      const long long ideal = (long long)base + (long long)((unsigned long long)cg * k / G);
      const long long lim = (long long)((unsigned long long)cg / (2ull * G));
      const long long t = ideal - max(-lim, min(lim, err));
      const int s0 = g ? n1 : 0, s1 = g ? n : n1;
      const int c = block_at(pref, nt, s0, s1, bpe, (unsigned)t, pb, sig);
      err += (long long)cost_before(pref, nt, c, bpe, pb, sig) - ideal;
      cut[q] = c;
    }
  }
  // lane q < 8 returns the cut of range q >> 1 at bound q & 1
  int r = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int v = __shfl_sync(kFull, cut[q], lane & 1);
    if ((lane >> 1) == q) r = v;
  }
  return r;
}

// 18 warps: 16 compute warps (two teams), a producer warp and a helper warp (see the top
// of this file).  RA / RB: the chunk rounds of phase A / B fixed at compile time (the
// widths the launch sees most, 4096 / 2048: 4 / 2), or 0 for any width (a run-time
// switch over the instances); XR = 1: the window's x rows are resident (the launch's
// x_res), so phase A has no activation sets, or -1: decided per window.  The fixed
// instances carry only the code their windows use.
template <int F, int RA = 0, int RB = 0, int XR = -1>
__global__ void __launch_bounds__(kThreads, 1) layer_kernel(const LayerArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  // window plan, set by warp 0 after the union: segments of phase A and B, ring depth,
  // resident x rows, the wide layout
  __shared__ int s_u, s_nsb, s_ns, s_xres, s_wide, s_sega;
  __shared__ int s_rng[8];  // this CTA's block ranges (plan_shares)
  __shared__ unsigned s_act_off, s_act_size;
  __shared__ unsigned s_bbase, s_bhalf;  // per-team phase-B set halves: offset, size
  __shared__ int s_bsep;                 // the halves do not overlap the x rows
  __shared__ volatile int s_abort;
  __shared__ volatile int s_pub;  // blocks published by the helper warp
  __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ __align__(8) uint64_t done[kPubRing];           // a block's outputs written
  __shared__ __align__(8) uint64_t set_in[1], set_out[1];    // activation-set hand-over
  __shared__ __align__(8) uint64_t team_in[kTeams], team_out[kTeams];  // per-team phase-B sets
  const LayerGeom& G = a.g;
  const int P = a.T * a.k;
  const LayerSmem L = layer_smem(a.E, P, a.logits != nullptr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned* exit_cnt = a.sync;
  unsigned* hdone = a.sync + 1;
  unsigned* ydone = a.sync + 1 + kMaxPairsFused;
  const unsigned stride_a = act_bytes(G.rounds_a), stride_b = act_bytes(G.rounds_b);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kTeamWarps);
    }
    for (int i = 0; i < kPubRing; ++i) mbar_init(&done[i], kTeamWarps);
    mbar_init(&set_in[0], kWarps);
    mbar_init(&set_out[0], kWarps);
    for (int t = 0; t < kTeams; ++t) {
      mbar_init(&team_in[t], kTeamWarps);
      mbar_init(&team_out[t], kTeamWarps);
    }
    s_abort = 0;
    s_pub = 0;
    fence_barrier_init();
  }
  if (a.wait_prior) grid_dep_wait();

  // ---- route-union (warp 0), segments, the window's plan, and the pair maps ----
  int* uniq = reinterpret_cast<int*>(smem + L.unique);
  int* offs = reinterpret_cast<int*>(smem + L.offsets);
  int* plist = reinterpret_cast<int*>(smem + L.pair_list);
  int* pos_of = reinterpret_cast<int*>(smem + L.pos_of);
  int* tok_of = reinterpret_cast<int*>(smem + L.tok_of);  // token of each pair position
  int* sa_slot = reinterpret_cast<int*>(smem + L.sa_slot);
  int* sa_pos = reinterpret_cast<int*>(smem + L.sa_pos);
  int* sa_nt = reinterpret_cast<int*>(smem + L.sa_nt);
  int* sb_slot = reinterpret_cast<int*>(smem + L.sb_slot);
  int* sb_pos = reinterpret_cast<int*>(smem + L.sb_pos);
  int* sb_nt = reinterpret_cast<int*>(smem + L.sb_nt);
  unsigned char* ring = smem + G.tables;
  // every thread but the producer warp's, numbered 0 .. kThreads - 33
  const int wt = warp < kWarps ? (int)threadIdx.x : (int)threadIdx.x - 32;
  // ---- the router step, when fused: warps 0 .. kRouteWarps-1 take one token each in
  // turn (router.cuh), staging its logits in the ring and activation area, which are
  // unused until the plan is made; the picks and weights stay in shared memory ----
  const bool routed = a.logits != nullptr;
  int* ridx = reinterpret_cast<int*>(smem + L.ridx);
  float* rw = reinterpret_cast<float*>(smem + L.rw);
  if (routed) {
    if (warp < kRouteWarps) {
      const unsigned stride = (5u * (unsigned)a.E + 15u) & ~15u;
      float* v = reinterpret_cast<float*>(ring + (size_t)warp * stride);
      unsigned char* taken = reinterpret_cast<unsigned char*>(v + a.E);
      for (int t = warp; t < a.T; t += kRouteWarps) {
        int pi;
        float pw;
        router_row(a.logits + (size_t)t * a.E, a.E, a.k, a.renorm, v, taken, lane, &pi, &pw);
        if (lane < a.k) {
          ridx[t * a.k + lane] = pi;
          rw[t * a.k + lane] = pw;
        }
      }
    }
    if (warp != kWarps) named_barrier(kBarWork, kThreads - 32);  // every warp but the producer
  }
  if (warp == 0) {
    int nv;
    const int u = warp_route_union(routed ? ridx : a.idx, P, a.E, reinterpret_cast<int*>(smem + L.cnt),
                                   reinterpret_cast<int*>(smem + L.rank), uniq, offs, plist, &nv);
    // the plan: a window whose x rows fit the normal activation area keeps them resident;
    // one with an expert of more pairs than that area holds x rows takes the wide layout
    // (all x rows resident, shallower ring) when the launch planned one; phase-A
    // segments are whole experts when x is resident, else as many pairs as the area
    // holds rows; phase-B segments as many pairs as the area holds h rows
    int maxn = 0;
    for (int i = lane; i < u; i += 32) maxn = max(maxn, offs[i + 1] - offs[i]);
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) maxn = max(maxn, __shfl_xor_sync(kFull, maxn, d));
    const int sega_n = (int)(G.act_n / stride_a);
    const bool wide = !a.x_res && G.stages_w >= 2 && maxn > sega_n;
    const bool xr = a.x_res || wide;
    const unsigned act_size = wide ? G.act_w : G.act_n;
    const int ns = wide ? G.stages_w : G.stages;
    const int sega = xr ? max(P, 1) : max(sega_n, 1);
    // phase-B sets are per team, each in half of the area; when the resident x rows
    // leave room for halves that hold as many pairs as an expert can have (at most T),
    // the halves follow the x rows, and no team waits for the other at the turn from
    // phase A to phase B
    const unsigned xbytes = xr ? (unsigned)(((size_t)a.T * stride_a + 15) & ~(size_t)15) : 0u;
    const unsigned half_all = (act_size / 2) & ~15u;
    const unsigned half_sep = xbytes < act_size ? ((act_size - xbytes) / 2) & ~15u : 0u;
    const int need = max(min(a.T, (int)(half_all / stride_b)), 1);
    const bool bsep = xr && (int)(half_sep / stride_b) >= need;
    const unsigned bhalf = bsep ? half_sep : half_all;
    const int segb = max((int)(bhalf / stride_b), 1);
    const int nsa = make_segments(offs, u, sega, sa_slot, sa_pos, sa_nt, lane);
    const int nsb = make_segments(offs, u, segb, sb_slot, sb_pos, sb_nt, lane);
    __syncwarp();
    // (the union's rank scratch and tok_of, filled only after the plan, hold the cost
    // prefixes)
    const int rq = plan_shares(sa_slot, sa_nt, nsa, a.I / kRowsA, sb_slot, sb_nt, nsb,
                               (a.H + G.rows_b - 1) / G.rows_b,
                               reinterpret_cast<unsigned*>(smem + L.rank),
                               reinterpret_cast<unsigned*>(tok_of), lane);
    if (lane < 8) s_rng[lane] = rq;
    if (lane == 0) {
      s_u = u;
      s_nsb = nsb;
      s_ns = ns;
      s_xres = xr ? 1 : 0;
      s_wide = wide ? 1 : 0;
      s_sega = sega;
      s_act_off = G.tables + (unsigned)ns * G.stage_bytes;
      s_act_size = act_size;
      s_bbase = bsep ? xbytes : 0u;
      s_bhalf = bhalf;
      s_bsep = bsep ? 1 : 0;
    }
    __syncwarp();
    named_barrier_arrive(kBarUnion, 64);  // the producer may start (it waits on this)
  } else if (warp != kWarps) {
    // compute warps 1.. and the helper: kThreads - 64 threads
    for (int p = wt - 32; p < P; p += kThreads - 64) pos_of[p] = -1;
    // a window whose x rows fit the normal activation area: converted while warp 0
    // forms the union
    if (a.x_res)
      convert_x_all<F>(a, G, smem + G.tables + (unsigned)G.stages * G.stage_bytes, wt - 32,
                       kThreads - 64, lane);
  }
  if (warp != kWarps) {
    named_barrier(kBarWork, kThreads - 32);  // every warp but the producer
  } else {
    named_barrier(kBarUnion, 64);  // the plan is made
  }
  const int u = s_u, nsb = s_nsb, NS = s_ns;
  const bool x_res = XR == 1 ? true : s_xres != 0;
  unsigned char* actp = smem + s_act_off;  // activation area (resident x rows first)
  const int n_valid = offs[u];
  if (warp != kWarps) {
    for (int i = wt; i < n_valid; i += kThreads - 32) {
      pos_of[plist[i]] = i;
      tok_of[i] = plist[i] / a.k;
    }
    if (s_wide) convert_x_all<F>(a, G, actp, wt, kThreads - 32, lane);  // wide: x now
    named_barrier(kBarWork, kThreads - 32);
  }

  if (blockIdx.x == 0 && warp == 2 && routed && a.ridx_out) {
    for (int i = lane; i < P; i += 32) {
      a.ridx_out[i] = ridx[i];
      a.rw_out[i] = rw[i];
    }
  }
  if (blockIdx.x == 0 && warp == 1 && a.ex_u) {
    for (int i = lane; i < u; i += 32) a.ex_unique[i] = uniq[i];
    for (int i = lane; i <= u; i += 32) a.ex_offsets[i] = offs[i];
    for (int i = lane; i < P; i += 32) a.ex_pair_list[i] = plist[i];
    if (lane == 0) *a.ex_u = u;
  }

  // ---- this CTA's blocks: phase-A blocks (kRowsA rows of gate and of up each, per
  // phase-A segment), then phase-B blocks (rows_b rows of down each, per phase-B
  // segment), each phase in two groups of experts, each group's share contiguous in
  // segment order and balanced by cost (plan_shares).  Every block is 2 kRowsA H/2 +
  // scales (A) or rows_b I/2 + scales (B) bytes; the two are equal at the 4096/2048
  // shape ----
  const int bpe_a = a.I / kRowsA;                     // phase-A blocks per segment
  const int bpe_b = (a.H + G.rows_b - 1) / G.rows_b;  // phase-B blocks per segment
  // the CTA's ranges (plan_shares): phase A group 1, group 2, phase B group 1, group 2
  const int a0 = s_rng[0], a2 = s_rng[2], b0 = s_rng[4], b2 = s_rng[6];
  const int nA1 = s_rng[1] - a0, nA = nA1 + (s_rng[3] - a2);
  const int nB1 = s_rng[5] - b0, nblk = nA + nB1 + (s_rng[7] - b2);
  // blk / bpe as a multiply-high by m = ceil(2^32 / bpe), exact while blk * bpe < 2^32
  // (here blk < 2^20 and 2 <= bpe <= 2^10)
  const unsigned mag_a = 0xFFFFFFFFu / (unsigned)bpe_a + 1u;
  const unsigned mag_b = 0xFFFFFFFFu / (unsigned)bpe_b + 1u;
  auto block_of = [&](int j, bool& pb, int& sg, int& row0) {
    if (j < nA) {
      const int blk = j < nA1 ? a0 + j : a2 + (j - nA1);
      pb = false;
      sg = (int)__umulhi((unsigned)blk, mag_a);
      row0 = (blk - sg * bpe_a) * kRowsA;
    } else {
      const int jb = j - nA;
      const int blk = jb < nB1 ? b0 + jb : b2 + (jb - nB1);
      pb = true;
      sg = (int)__umulhi((unsigned)blk, mag_b);
      row0 = (blk - sg * bpe_b) * G.rows_b;
    }
  };
  // block j starts an activation set: the first block of a segment (or of one of the
  // four ranges) in phase B, and in phase A when x is not resident
  auto set_start = [&](int j) -> bool {
    bool pb;
    int sg, r0;
    block_of(j, pb, sg, r0);
    if (!pb && x_res) return false;
    return r0 == 0 || j == 0 || j == nA1 || j == nA || j == nA + nB1;
  };

  if (warp == kWarps + 1) {
    // ================================ helper warp ================================
    // Publishes finished blocks in order: a phase-A block adds 1 to hdone of its expert
    // (its h rows written), a phase-B block adds 1 to ydone of its row block.  The
    // compute warps' done arrivals released their stores at CTA scope and the test
    // below acquires them; the device-scope release reductions pass them on
    // (causality order is transitive across the two scopes).  All the finished blocks
    // found in one pass go out behind one device-scope fence (a fence followed by
    // relaxed reductions releases each of them), and consecutive blocks of one counter
    // add together: one fence and a few reductions per pass, however many blocks.
    unsigned long long t_prog = globaltimer();
    for (int j = 0; j < nblk;) {
      int n = 0;
      while (j + n < nblk && n < kPubRing &&
             lane0(mbar_test(&done[(j + n) % kPubRing], ((j + n) / kPubRing) & 1)))
        ++n;
      if (n > 0) {
        if (lane == 0) {
          fence_acq_rel_gpu();
          unsigned* cur = nullptr;
          unsigned cnt = 0;
          for (int q = j; q < j + n; ++q) {
            bool pb;
            int sg, row0;
            block_of(q, pb, sg, row0);
            unsigned* c = pb ? &ydone[row0 / G.rows_b] : &hdone[sa_slot[sg]];
            if (c != cur) {
              if (cnt) red_relaxed_gpu(cur, cnt);
              cur = c;
              cnt = 0;
            }
            ++cnt;
          }
          red_relaxed_gpu(cur, cnt);
          s_pub = j + n;
        }
        __syncwarp();
        j += n;
        t_prog = globaltimer();
      } else {
        if (lane0(s_abort != 0)) break;
        if (lane0(globaltimer() - t_prog > wait_limit())) {
          if (lane == 0) {
            set_error(kErrTimeout);
            s_abort = 1;
          }
          break;
        }
        // suspended (not spinning on issue slots) until block j is done, or briefly
        mbar_try_wait(&done[j % kPubRing], (j / kPubRing) & 1);
      }
    }
  } else if (warp == kWarps) {
    // =============================== producer warp ===============================
    // Issues this CTA's blocks into the stage ring, in order.  Every condition is lane
    // 0's (uniform control flow).
    auto timed_out = [&](unsigned long long t0) -> bool {
      if (lane0(s_abort != 0)) return true;
      if (lane0(globaltimer() - t0 > wait_limit())) {
        if (lane == 0) {
          set_error(kErrTimeout);
          s_abort = 1;
        }
        return true;
      }
      return false;
    };
    bool ok = true;
    int j = 0;
    for (; j < nblk && ok; ++j) {
      const int st = j % NS;
      if (j >= NS) {  // the compute warps are done with block j - NS
        const unsigned long long t0 = globaltimer();
        // (try_wait suspends the warp, leaving the issue slots to the compute warps)
        while (!lane0(mbar_try_wait(&empty[st], ((j / NS) - 1) & 1)))
          if (timed_out(t0)) {
            ok = false;
            break;
          }
      }
      {  // block j's publication barrier is free: block j - kPubRing was published
        const unsigned long long t0 = globaltimer();
        while (ok && lane0_int(s_pub) <= j - kPubRing) {
          if (timed_out(t0)) ok = false;
          __nanosleep(32);
        }
      }
      if (!ok) break;
      bool pb;
      int sg, row0;
      block_of(j, pb, sg, row0);
      if (lane == 0) {
        unsigned char* buf = ring + (size_t)st * G.stage_bytes;
        fence_proxy_async();
        if (!pb) {
          const size_t r0 = (size_t)uniq[sa_slot[sg]] * a.I + row0;
          const size_t qrow = a.H / 8, srow = a.H / 64;
          mbar_arrive_expect_tx(&full[st], G.a_bytes);
          bulk_g2s_stream(buf, a.gq + r0 * qrow, G.a_q, &full[st]);
          bulk_g2s_stream(buf + G.a_q, a.gs + r0 * srow, G.a_sb, &full[st]);
          if (F != kFmtMx) bulk_g2s_stream(buf + G.a_q + G.a_sb, a.gb + r0 * srow, G.a_sb, &full[st]);
          buf += G.a_mat;
          bulk_g2s_stream(buf, a.uq + r0 * qrow, G.a_q, &full[st]);
          bulk_g2s_stream(buf + G.a_q, a.us + r0 * srow, G.a_sb, &full[st]);
          if (F != kFmtMx) bulk_g2s_stream(buf + G.a_q + G.a_sb, a.ub + r0 * srow, G.a_sb, &full[st]);
        } else {
          const int nrows = min(G.rows_b, a.H - row0);
          const size_t r0 = (size_t)uniq[sb_slot[sg]] * a.H + row0;
          const size_t qrow = a.I / 8, srow = a.I / 64;
          const unsigned qb = nrows * (a.I / 2), sb = nrows * (a.I / 32);
          mbar_arrive_expect_tx(&full[st], qb + (F == kFmtMx ? 1 : 2) * sb);
          bulk_g2s_stream(buf, a.dq + r0 * qrow, qb, &full[st]);
          bulk_g2s_stream(buf + G.b_q, a.ds + r0 * srow, sb, &full[st]);
          if (F != kFmtMx) bulk_g2s_stream(buf + G.b_q + G.b_sb, a.db + r0 * srow, sb, &full[st]);
        }
      }
      __syncwarp();
    }
    // copies still in flight after an abort land before the CTA exits (bounded)
    if (!ok && lane == 0) {
      const int issued = j < nblk ? j : nblk;
      for (int g = (issued > NS ? issued - NS : 0); g < issued; ++g) {
        const unsigned long long t0 = globaltimer();
        while (!mbar_test(&full[g % NS], (g / NS) & 1) && globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
    __syncwarp();
  } else {
    // ================================ compute warps ================================
    // Two teams of kTeamWarps warps: team tm takes blocks tm, tm + kTeams, ... of this
    // CTA's sequence, warp w of a team row w of each of its blocks (phase A) or rows
    // w, w + kTeamWarps, ... (phase B).  While one team computes a block the other
    // computes the next, so each scheduler has twice the warps to hide latency with.
    const int tm = warp / kTeamWarps, w = warp % kTeamWarps;
    auto wait_cons = [&](uint64_t* bar, unsigned parity) -> bool {
      if (s_abort) return false;
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(bar, parity)) {
        if (s_abort) return false;
        if (globaltimer() - t0 > wait_limit()) {
          set_error(kErrTimeout);
          s_abort = 1;
          return false;
        }
      }
      return true;
    };
    const int sega = s_sega;
    int nsets = 0;    // all-warp meetings at set starts
    int nteam = 0;    // this team's phase-B sets converted
    int handled = -1; // blocks up to here have had their set starts taken
    // this team's phase-B set buffer: half the activation area
    unsigned char* bset = actp + s_bbase + (size_t)tm * s_bhalf;
    const bool bsep = s_bsep != 0;
    // Set starts, in block order, before a block at or after them is computed.
    // Phase A (x not resident): every compute warp takes it; all meet at set_in (the
    // previous set's blocks are done, the area is free), the 512 compute threads
    // convert the x rows into the area, and all meet at set_out.
    // Phase B: each team keeps its own copy of the set's h rows in its half of the area,
    // so the teams do not wait for each other; the first phase-B set start is also an
    // all-warp meeting when the halves overlap the x rows or phase-A sets.  One thread
    // per team waits (bounded, with back-off) until hdone[expert] counts every phase-A
    // block of the expert, its acquire reaching the team's warps through team_in, then
    // the team's 256 threads convert the rows and meet at team_out.
    auto take_sets = [&](int upto) -> bool {
      for (int b = handled + 1; b <= upto; ++b) {
        if (!set_start(b)) continue;
        bool pb;
        int sg, r0;
        block_of(b, pb, sg, r0);
        const int nt = pb ? sb_nt[sg] : sa_nt[sg];
        const int p0 = pb ? sb_pos[sg] : sa_pos[sg];
        if constexpr (XR != 1) {
          if (!pb) {  // phase-A set (x not resident): all-warp meeting and conversion
            __syncwarp();
            if (lane == 0) mbar_arrive(&set_in[0]);
            if (!wait_cons(&set_in[0], nsets & 1)) return false;
            convert_set<F>(a, G, false, tok_of, p0, nt, actp, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&set_out[0]);
            if (!wait_cons(&set_out[0], nsets & 1)) return false;
            ++nsets;
            continue;
          }
        }
        if (b == nA && !bsep) {  // the turn to phase B over the x rows: all-warp meeting
          __syncwarp();
          if (lane == 0) mbar_arrive(&set_in[0]);
          if (!wait_cons(&set_in[0], nsets & 1)) return false;
          ++nsets;
        }
        __syncwarp();
        if (w == 0 && lane == 0) {
          const int slot = sb_slot[sg];
          const int n_i = offs[slot + 1] - offs[slot];
          const unsigned target = (unsigned)bpe_a * (unsigned)((n_i + sega - 1) / sega);
          const unsigned long long t0 = globaltimer();
          while (!s_abort && ld_acquire_gpu(&hdone[slot]) < target) {
            if (globaltimer() - t0 > wait_limit()) {
              set_error(kErrTimeout);
              s_abort = 1;
            }
            __nanosleep(32);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&team_in[tm]);
        if (!wait_cons(&team_in[tm], nteam & 1)) return false;
        convert_set<F>(a, G, true, tok_of, p0, nt, bset, lane, w * 32 + lane, kTeamWarps * 32);
        __syncwarp();
        if (lane == 0) mbar_arrive(&team_out[tm]);
        if (!wait_cons(&team_out[tm], nteam & 1)) return false;
        ++nteam;
      }
      handled = upto;
      return true;
    };
    // this warp is done reading stage st, and its outputs of block jb are written
    // (released at CTA scope)
    auto finish = [&](int st, int jb) {
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[st]);
        mbar_arrive(&done[jb % kPubRing]);
      }
    };
    // the phase-A blocks, then the phase-B blocks, in two loops (each loop's code holds
    // only its phase's core)
    int j = tm;
    bool go = true;
    for (; j < nA; j += kTeams) {
      if (!take_sets(j)) {
        go = false;
        break;
      }
      const int st = j % NS;
      if (!wait_cons(&full[st], (j / NS) & 1)) {
        go = false;
        break;
      }
      bool phase_b;
      int sg, row0;
      block_of(j, phase_b, sg, row0);
      const int nt = sa_nt[sg];
      const int p0 = sa_pos[sg];
      const unsigned char* buf = ring + (size_t)st * G.stage_bytes;
      const unsigned char* bgq = buf + (size_t)w * (a.H / 2);
      const uint16_t* bgs = reinterpret_cast<const uint16_t*>(buf + G.a_q) + w * (a.H / 64);
      const uint16_t* bgb = reinterpret_cast<const uint16_t*>(buf + G.a_q + G.a_sb) + w * (a.H / 64);
      const unsigned char* bu = buf + G.a_mat;
      const unsigned char* buq = bu + (size_t)w * (a.H / 2);
      const uint16_t* bus = reinterpret_cast<const uint16_t*>(bu + G.a_q) + w * (a.H / 64);
      const uint16_t* bub = reinterpret_cast<const uint16_t*>(bu + G.a_q + G.a_sb) + w * (a.H / 64);
      // the segment's pairs two at a time (the codes split once for both), the last one
      // alone; the block's weights read again per pass
      for (int c = 0; c < nt; c += kNT) {
        const int ntc = min(kNT, nt - c);
        // each pair's activation row: the token's resident x row, or its row of the set
        const unsigned char* arow[kNT];
#pragma unroll
        for (int t = 0; t < kNT; ++t) {
          const int q = c + (t < ntc ? t : 0);
          arow[t] = x_res ? actp + tok_of[p0 + q] * stride_a : actp + q * stride_a;
        }
        float Gs[kNT], Us[kNT];
        if constexpr (RA > 0) {
          if (ntc == 2) rows_a<2, RA, F>(bgq, bgs, bgb, buq, bus, bub, a.H, arow, lane, Gs, Us);
          else rows_a<1, RA, F>(bgq, bgs, bgb, buq, bus, bub, a.H, arow, lane, Gs, Us);
        } else {
          if (ntc == 2) dispatch_a<2, F>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, arow, lane, Gs, Us);
          else dispatch_a<1, F>(G.rounds_a, bgq, bgs, bgb, buq, bus, bub, a.H, arow, lane, Gs, Us);
        }
        if (lane < ntc) {
          const float g = round_to_bf16(lane == 0 ? Gs[0] : Gs[1]);
          const float hu = round_to_bf16(lane == 0 ? Us[0] : Us[1]);
          // silu(g) = g / (1 + e^-g); the fast division's error (2 ulp of fp32) is far
          // below the bf16 step h is rounded to
          a.h[(size_t)(p0 + c + lane) * a.I + row0 + w] =
              float_to_bf16_bits(__fdividef(g, 1.0f + __expf(-g)) * hu);
        }
      }
      finish(st, j);
    }
    for (; go && j < nblk; j += kTeams) {
      if (!take_sets(j)) {
        go = false;
        break;
      }
      const int st = j % NS;
      if (!wait_cons(&full[st], (j / NS) & 1)) {
        go = false;
        break;
      }
      bool phase_b;
      int sg, row0;
      block_of(j, phase_b, sg, row0);
      const int nt = sb_nt[sg];
      const int p0 = sb_pos[sg];
      const unsigned char* buf = ring + (size_t)st * G.stage_bytes;
      const int nrows = min(G.rows_b, a.H - row0);
      const uint16_t* bs = reinterpret_cast<const uint16_t*>(buf + G.b_q);
      const uint16_t* bb = reinterpret_cast<const uint16_t*>(buf + G.b_q + G.b_sb);
      // the segment's pairs one at a time, the block's weights read again per pair
      for (int c = 0; c < nt; ++c) {
        int vid;
        float v;
        if constexpr (RB > 0)
          v = rows_b<1, RB, F>(buf, bs, bb, w, nrows, a.I, bset + (size_t)c * stride_b,
                               stride_b, lane, vid);
        else
          v = dispatch_b<1, F>(G.rounds_b, buf, bs, bb, w, nrows, a.I,
                               bset + (size_t)c * stride_b, stride_b, lane, vid);
        if (vid >= 0) {
          const int r = w + kTeamWarps * (vid / kNT);
          if (r < nrows) a.y[(size_t)(p0 + c) * a.H + row0 + r] = v;
        }
      }
      finish(st, j);
    }
    if (go) take_sets(nblk - 1);  // the set starts past this team's last block
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
        while (!s_abort && ld_acquire_gpu(&ydone[rb]) < (unsigned)nsb) {
          if (globaltimer() - t0 > wait_limit()) {
            set_error(kErrTimeout);
            s_abort = 1;
          }
          __nanosleep(32);
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
            if (pos >= 0)
              acc = fmaf(routed ? rw[p] : __ldg(a.w + p), __ldcg(a.y + (size_t)pos * a.H + c), acc);
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
      for (int i = 0; i < u; ++i) hdone[i] = 0;
      *exit_cnt = 0;
      __threadfence();
    }
  }
}

}  // namespace qeg
