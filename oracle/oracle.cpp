// Oracle for the union-of-experts quantized SwitchGLU layer: a plain, slow,
// fp64 CPU implementation of what the layer computes.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// cpu_baseline / reference legs of bench.py may load it.  It shares no code
// with the CUDA library (quantized_expert_gather_b200/csrc) and includes none
// of its headers.
//
// What it follows:
// * SwitchGLU per (token, expert) pair, in the order of the moe_bench.py script
//   of "gather_qmm at M=1 streams 4-bit expert weights at ~half the bandwidth
//   of M=4" (mlx issue 4509, "Script"): up = W_up x, gate = W_gate x,
//   h = silu(gate) * up, y = W_down h.  Weights are mx.quantize'd with group
//   64, 4 bits, affine ("Numbers"): w = scale * q + bias per group of 64
//   input columns, scale and bias in bf16.
// * The gate and up results are bf16 tensors in that script, and the fused
//   gate+up tile of "Apple7/8 MoE gate and up in one decode pass" (splash
//   PR 45, "What changed") writes bf16(up) * silu(gate) from the bf16 gate.
//   Reading used here: g = bf16(G), v = bf16(U), h = bf16(g * sigmoid(g) * v)
//   with one rounding of the product; y stays unrounded through the combine.
// * Top-k combine: out[t] = sum_j w[t,j] * y[t,j] (the router weights are
//   taken as given).
// * Union of experts ("Small-L fused expert gather", mlx discussion 3801,
//   first post, "Two implications" item 1, and the grouped-GEMM framing of the
//   second post): the distinct experts of the window, ascending; each one's
//   (token, expert) pairs p = t*k + j in ascending p; offsets = exclusive
//   prefix of the per-expert pair counts.
// * Packing (the pages are silent): element c of a row is nibble c % 8 (bits
//   4*(c%8) .. 4*(c%8)+3, least significant first) of 32-bit word c / 8.
// * Expert ids outside [0, E) name no expert: such a pair is left out of the
//   union and contributes nothing.
// * mxfp4 banks (oracle_switchglu_mxfp4): GLM-5.2's routed banks are "mxfp4 gs32"
//   ("Small-L fused expert gather", mlx discussion 3801, the decomposition post).
//   Reading: the OCP microscaling format, e2m1 elements (values 0, 0.5, 1, 1.5,
//   2, 3, 4, 6 and their negatives) with one e8m0 scale 2^(e - 127) per 32
//   input columns, packed like the affine codes; w = e2m1(q) * 2^(e - 127).
// * The router step before the layer (oracle_router_topk): top-k of softmax over
//   the experts, renormalised over the k, as the tiny parity configuration routes
//   its tokens; equal logits go to the lower expert id.
//
// Every sum is in fp64 in ascending index order; dequantised weights are exact
// in fp64.  Rounding to bf16 is done directly from fp64 (one rounding).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <thread>
#include <vector>

namespace {

double bf16_value(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// Round an fp64 value to the nearest bf16 value (ties to even), returned in
// fp64.  bf16 keeps 8 significant bits; its smallest subnormal is 2^-133 and
// its largest finite value 255 * 2^120.
double round_bf16(double v) {
  if (v == 0.0 || !std::isfinite(v)) return v;
  int e;
  std::frexp(v, &e);  // |v| = m * 2^e with 0.5 <= m < 1
  int qexp = e - 8;
  if (qexp < -133) qexp = -133;
  const double r = std::ldexp(std::nearbyint(std::ldexp(v, -qexp)), qexp);
  if (std::fabs(r) > std::ldexp(255.0, 120)) return v > 0 ? INFINITY : -INFINITY;
  return r;
}

double sigmoid(double g) { return 1.0 / (1.0 + std::exp(-g)); }

// fp4 e2m1 code -> value: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0
// (the element format of mxfp4).
const double kE2M1[16] = {0.0,  0.5,  1.0,  1.5,  2.0,  3.0,  4.0,  6.0,
                          -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0};

// e8m0 scale byte -> 2^(byte - 127) (the block scale of mxfp4; 255 would be NaN).
double e8m0_value(uint8_t v) { return std::ldexp(1.0, static_cast<int>(v) - 127); }

struct Matrix {  // one expert bank, q [E, rows, cols/8] and per format:
  const uint32_t* q;
  const uint16_t* s;   // affine group 64: scales bf16 [E, rows, cols/64]
  const uint16_t* b;   //                  biases bf16 [E, rows, cols/64]
  const uint8_t* e8;   // mxfp4 group 32: e8m0 scales [E, rows, cols/32]
  int rows, cols;
  bool mxfp4;
  // dequantised weight of expert e at (row, col)
  double at(int e, int row, int col) const {
    const size_t r = static_cast<size_t>(e) * rows + row;
    const uint32_t word = q[r * (cols / 8) + col / 8];
    const int nib = static_cast<int>((word >> (4 * (col % 8))) & 0xFu);
    if (mxfp4) return kE2M1[nib] * e8m0_value(e8[r * (cols / 32) + col / 32]);
    const size_t g = r * (cols / 64) + col / 64;
    return bf16_value(s[g]) * nib + bf16_value(b[g]);
  }
};

struct Layer {
  const uint16_t* x;   // [T, H] bf16 bits
  const int32_t* idx;  // [T, k]
  const float* w;      // [T, k]
  Matrix gate, up, down;
  int T, k, E, H, I;
};

bool valid_expert(const Layer& L, int e) { return e >= 0 && e < L.E; }

// h for rows [r0, r1) of pair p: G, U, then the bf16 readings above.
void pair_h_rows(const Layer& L, int p, int r0, int r1, double* h) {
  const int t = p / L.k, e = L.idx[p];
  const uint16_t* x = L.x + static_cast<size_t>(t) * L.H;
  for (int r = r0; r < r1; ++r) {
    double G = 0.0, U = 0.0;
    for (int c = 0; c < L.H; ++c) {
      const double xc = bf16_value(x[c]);
      G += L.gate.at(e, r, c) * xc;
      U += L.up.at(e, r, c) * xc;
    }
    const double g = round_bf16(G), v = round_bf16(U);
    h[r] = round_bf16(g * sigmoid(g) * v);
  }
}

// y for rows [c0, c1) of pair p from its h.
void pair_y_rows(const Layer& L, int p, int c0, int c1, const double* h, double* y) {
  const int e = L.idx[p];
  for (int c = c0; c < c1; ++c) {
    double Y = 0.0;
    for (int r = 0; r < L.I; ++r) Y += L.down.at(e, c, r) * h[r];
    y[c] = Y;
  }
}

// Run task(i) for i in [0, n) on up to n_threads threads.  Each task writes
// disjoint outputs, so the result does not depend on the thread count.
template <class F>
void parallel_for(int n, int n_threads, F task) {
  if (n_threads <= 1 || n <= 1) {
    for (int i = 0; i < n; ++i) task(i);
    return;
  }
  std::atomic<int> next(0);
  std::vector<std::thread> pool;
  const int nt = std::min(n_threads, n);
  for (int i = 0; i < nt; ++i)
    pool.emplace_back([&]() {
      for (int j = next++; j < n; j = next++) task(j);
    });
  for (auto& th : pool) th.join();
}

Layer make_layer(const uint16_t* x, const int32_t* idx, const float* w, const uint32_t* gq,
                 const uint16_t* gs, const uint16_t* gb, const uint32_t* uq, const uint16_t* us,
                 const uint16_t* ub, const uint32_t* dq, const uint16_t* ds, const uint16_t* db,
                 int T, int k, int E, int H, int I) {
  Layer L;
  L.x = x; L.idx = idx; L.w = w;
  L.gate = Matrix{gq, gs, gb, nullptr, I, H, false};
  L.up = Matrix{uq, us, ub, nullptr, I, H, false};
  L.down = Matrix{dq, ds, db, nullptr, H, I, false};
  L.T = T; L.k = k; L.E = E; L.H = H; L.I = I;
  return L;
}

// Pairs of the selected tokens (all tokens when tokens == nullptr), ascending.
std::vector<int> selected_pairs(const Layer& L, const int32_t* tokens, int n_tokens) {
  std::vector<int> pairs;
  if (!tokens) {
    for (int p = 0; p < L.T * L.k; ++p) pairs.push_back(p);
  } else {
    std::vector<int> ts(tokens, tokens + n_tokens);
    std::sort(ts.begin(), ts.end());
    ts.erase(std::unique(ts.begin(), ts.end()), ts.end());
    for (int t : ts)
      for (int j = 0; j < L.k; ++j) pairs.push_back(t * L.k + j);
  }
  return pairs;
}

void combine(const Layer& L, const std::vector<int>& pairs, const std::vector<double>& Y,
             double* out) {
  // out[t, c] = sum over j (ascending) of w[t, j] * y[t, j][c]; invalid pairs skipped.
  std::map<int, std::vector<int>> by_token;
  for (size_t i = 0; i < pairs.size(); ++i) by_token[pairs[i] / L.k].push_back(static_cast<int>(i));
  for (auto& kv : by_token) {
    double* o = out + static_cast<size_t>(kv.first) * L.H;
    for (int c = 0; c < L.H; ++c) {
      double acc = 0.0;
      for (int i : kv.second) {
        const int p = pairs[i];
        if (!valid_expert(L, L.idx[p])) continue;
        acc += static_cast<double>(L.w[p]) * Y[static_cast<size_t>(i) * L.H + c];
      }
      o[c] = acc;
    }
  }
}

}  // namespace

namespace {
void run_switchglu(const Layer& L, const int32_t* tokens, int n_tokens, int n_threads,
                   double* out, double* h_out, double* y_out);
}  // namespace

extern "C" {

// Route-union by its plain definition.  unique[min(E,P)], offsets[min(E,P)+1],
// pair_list[P]; entries of pair_list past offsets[u] are set to -1.
// Returns the number of pairs whose expert id is outside [0, E).
int oracle_route_union(const int32_t* idx, int T, int k, int E, int32_t* unique,
                       int32_t* offsets, int32_t* pair_list, int32_t* num_unique) {
  const int P = T * k;
  std::map<int, std::vector<int>> groups;  // expert -> its pairs, ascending p
  int invalid = 0;
  for (int p = 0; p < P; ++p) {
    const int e = idx[p];
    if (e < 0 || e >= E) {
      ++invalid;
      continue;
    }
    groups[e].push_back(p);
  }
  int slot = 0, pos = 0;
  for (auto& kv : groups) {
    unique[slot] = kv.first;
    offsets[slot] = pos;
    for (int p : kv.second) pair_list[pos++] = p;
    ++slot;
  }
  offsets[slot] = pos;
  for (int i = pos; i < P; ++i) pair_list[i] = -1;
  *num_unique = slot;
  return invalid;
}

// Per-pair definition (no deduplication).  out [T, H] fp64: rows of the
// selected tokens are written (all rows when tokens == nullptr).  h_out
// [T*k, I] (optional): the bf16-rounded h of every selected pair, indexed by
// p = t*k + j; rows of invalid pairs are zero.  y_out [T*k, H] (optional): y of
// every selected pair.
void oracle_switchglu(const uint16_t* x, const int32_t* idx, const float* w, const uint32_t* gq,
                      const uint16_t* gs, const uint16_t* gb, const uint32_t* uq,
                      const uint16_t* us, const uint16_t* ub, const uint32_t* dq,
                      const uint16_t* ds, const uint16_t* db, int T, int k, int E, int H, int I,
                      const int32_t* tokens, int n_tokens, int n_threads, double* out,
                      double* h_out, double* y_out) {
  run_switchglu(make_layer(x, idx, w, gq, gs, gb, uq, us, ub, dq, ds, db, T, k, E, H, I),
                tokens, n_tokens, n_threads, out, h_out, y_out);
}

// The same layer on mxfp4 banks (group 32): q [E, rows, cols/8] e2m1 codes packed
// as above, e8 [E, rows, cols/32] e8m0 scales; w = e2m1(q) * 2^(e8 - 127).
void oracle_switchglu_mxfp4(const uint16_t* x, const int32_t* idx, const float* w,
                            const uint32_t* gq, const uint8_t* ge8, const uint32_t* uq,
                            const uint8_t* ue8, const uint32_t* dq, const uint8_t* de8, int T,
                            int k, int E, int H, int I, const int32_t* tokens, int n_tokens,
                            int n_threads, double* out, double* h_out, double* y_out) {
  Layer L;
  L.x = x; L.idx = idx; L.w = w;
  L.gate = Matrix{gq, nullptr, nullptr, ge8, I, H, true};
  L.up = Matrix{uq, nullptr, nullptr, ue8, I, H, true};
  L.down = Matrix{dq, nullptr, nullptr, de8, H, I, true};
  L.T = T; L.k = k; L.E = E; L.H = H; L.I = I;
  run_switchglu(L, tokens, n_tokens, n_threads, out, h_out, y_out);
}

// One mxfp4 weight, exported so its pins can test the decoding directly.
double oracle_mxfp4_value(int code, int scale) {
  return kE2M1[code & 15] * e8m0_value(static_cast<uint8_t>(scale));
}

}  // extern "C"

namespace {

void run_switchglu(const Layer& L, const int32_t* tokens, int n_tokens, int n_threads,
                   double* out, double* h_out, double* y_out) {
  const int T = L.T, k = L.k, E = L.E, H = L.H, I = L.I;
  (void)T; (void)k; (void)E;
  const std::vector<int> pairs = selected_pairs(L, tokens, n_tokens);
  const int np = static_cast<int>(pairs.size());
  std::vector<double> hbuf(static_cast<size_t>(np) * I, 0.0), ybuf(static_cast<size_t>(np) * H, 0.0);
  const int RB = 64;  // rows per task
  const int nbi = (I + RB - 1) / RB, nbh = (H + RB - 1) / RB;
  parallel_for(np * nbi, n_threads, [&](int task) {
    const int i = task / nbi, blk = task % nbi;
    if (!valid_expert(L, L.idx[pairs[i]])) return;
    pair_h_rows(L, pairs[i], blk * RB, std::min(I, (blk + 1) * RB), &hbuf[static_cast<size_t>(i) * I]);
  });
  parallel_for(np * nbh, n_threads, [&](int task) {
    const int i = task / nbh, blk = task % nbh;
    if (!valid_expert(L, L.idx[pairs[i]])) return;
    pair_y_rows(L, pairs[i], blk * RB, std::min(H, (blk + 1) * RB), &hbuf[static_cast<size_t>(i) * I],
                &ybuf[static_cast<size_t>(i) * H]);
  });
  combine(L, pairs, ybuf, out);
  for (int i = 0; i < np; ++i) {
    if (h_out)
      std::memcpy(h_out + static_cast<size_t>(pairs[i]) * I, &hbuf[static_cast<size_t>(i) * I],
                  sizeof(double) * I);
    if (y_out)
      std::memcpy(y_out + static_cast<size_t>(pairs[i]) * H, &ybuf[static_cast<size_t>(i) * H],
                  sizeof(double) * H);
  }
}

}  // namespace

extern "C" {

// Deduplicated form: take the union of experts, dequantise each distinct
// expert's three matrices once, and apply them to every pair routed to it
// (ascending expert, ascending p).  Each pair's arithmetic is the same as in
// oracle_switchglu, so the result must be identical bit for bit.
void oracle_switchglu_union(const uint16_t* x, const int32_t* idx, const float* w,
                            const uint32_t* gq, const uint16_t* gs, const uint16_t* gb,
                            const uint32_t* uq, const uint16_t* us, const uint16_t* ub,
                            const uint32_t* dq, const uint16_t* ds, const uint16_t* db, int T,
                            int k, int E, int H, int I, double* out, double* h_out) {
  const Layer L = make_layer(x, idx, w, gq, gs, gb, uq, us, ub, dq, ds, db, T, k, E, H, I);
  const int P = T * k;
  std::vector<int32_t> uniq(std::max(1, std::min(E, P))), offs(std::max(1, std::min(E, P)) + 1),
      plist(std::max(1, P));
  int32_t u = 0;
  oracle_route_union(idx, T, k, E, uniq.data(), offs.data(), plist.data(), &u);
  std::vector<double> Y(static_cast<size_t>(P) * H, 0.0), hv(static_cast<size_t>(P) * I, 0.0);
  std::vector<double> Wg(static_cast<size_t>(I) * H), Wu(static_cast<size_t>(I) * H),
      Wd(static_cast<size_t>(H) * I);
  for (int s = 0; s < u; ++s) {
    const int e = uniq[s];
    for (int r = 0; r < I; ++r)
      for (int c = 0; c < H; ++c) {
        Wg[static_cast<size_t>(r) * H + c] = L.gate.at(e, r, c);
        Wu[static_cast<size_t>(r) * H + c] = L.up.at(e, r, c);
      }
    for (int c = 0; c < H; ++c)
      for (int r = 0; r < I; ++r) Wd[static_cast<size_t>(c) * I + r] = L.down.at(e, c, r);
    for (int i = offs[s]; i < offs[s + 1]; ++i) {
      const int p = plist[i], t = p / k;
      double* h = &hv[static_cast<size_t>(p) * I];
      for (int r = 0; r < I; ++r) {
        double G = 0.0, U = 0.0;
        for (int c = 0; c < H; ++c) {
          const double xc = bf16_value(x[static_cast<size_t>(t) * H + c]);
          G += Wg[static_cast<size_t>(r) * H + c] * xc;
          U += Wu[static_cast<size_t>(r) * H + c] * xc;
        }
        const double g = round_bf16(G), v = round_bf16(U);
        h[r] = round_bf16(g * sigmoid(g) * v);
      }
      for (int c = 0; c < H; ++c) {
        double acc = 0.0;
        for (int r = 0; r < I; ++r) acc += Wd[static_cast<size_t>(c) * I + r] * h[r];
        Y[static_cast<size_t>(p) * H + c] = acc;
      }
    }
  }
  for (int t = 0; t < T; ++t)
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) {
        const int p = t * k + j;
        if (!valid_expert(L, idx[p])) continue;
        acc += static_cast<double>(w[p]) * Y[static_cast<size_t>(p) * H + c];
      }
      out[static_cast<size_t>(t) * H + c] = acc;
    }
  if (h_out) std::memcpy(h_out, hv.data(), sizeof(double) * hv.size());
}

// The oracle's bf16 rounding, exported so its pins can test it directly.
double oracle_round_bf16(double v) { return round_bf16(v); }

// Router step ahead of the layer, by its plain definition (the routing of the
// tiny parity configuration: top-k of softmax over the E experts, weights
// renormalised over the k).  For each token t: the k experts with the largest
// logits, in descending logit order with the lower expert id first among equal
// logits; w_j = exp(l_j - m) / D with m the row's largest logit and D the sum of
// exp(l - m) over the k chosen experts (renormalize != 0) or over all E.
// Logits are finite; sums in fp64, ascending order.
void oracle_router_topk(const float* logits, int T, int E, int k, int renormalize,
                        int32_t* idx, double* w) {
  std::vector<int> order(E);
  for (int t = 0; t < T; ++t) {
    const float* row = logits + static_cast<size_t>(t) * E;
    for (int e = 0; e < E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(),
                     [row](int a, int b) { return row[a] > row[b]; });
    const double m = row[order[0]];
    double denom = 0.0;
    if (renormalize) {
      for (int j = 0; j < k; ++j) denom += std::exp(static_cast<double>(row[order[j]]) - m);
    } else {
      for (int e = 0; e < E; ++e) denom += std::exp(static_cast<double>(row[e]) - m);
    }
    for (int j = 0; j < k; ++j) {
      idx[static_cast<size_t>(t) * k + j] = order[j];
      w[static_cast<size_t>(t) * k + j] =
          std::exp(static_cast<double>(row[order[j]]) - m) / denom;
    }
  }
}

}  // extern "C"
