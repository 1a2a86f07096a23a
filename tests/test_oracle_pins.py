"""Pins for the fp64 oracle: things fixed by the pages and by mathematics, not by
the oracle itself.

* closed forms worked out by hand (tests/golden/closed_forms.txt);
* bf16 rounding against torch's fp32 -> bf16 conversion (a library routine);
* the route-union against brute force (Python sets and sorts);
* the deduplicated form equals the per-pair form bit for bit;
* invariants: router-weight scaling, slot permutation, zero weights, token
  independence;
* E=1, k=1 reduces to a dense dequantised GEMV -> SwiGLU -> GEMV done with numpy
  matmul (library routine);
* the router step: equal logits (ties to the lower id, weights 1/k or 1/E), a
  logarithmic ramp (weights proportional to i + 1, a closed form), k = E against
  scipy's softmax, torch.topk's selection, shift invariance;
* mxfp4 banks: the e2m1 / e8m0 decoding against ml_dtypes (a library routine), the
  layer on weights that both formats hold exactly bit-identical to the affine form,
  and E=1, k=1 against a dense SwiGLU of ml_dtypes-decoded matrices;
* a set of planted mistakes (in copies of the oracle source) each fail a pin.
"""
import math
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.layers import draw_bank, make_layer, read_golden, tiny_layer

GOLD = read_golden("closed_forms.txt")


# ---------------------------------------------------------------- helpers ---
def pack_nibbles(qmat: np.ndarray) -> np.ndarray:
    """[rows, cols] ints in 0..15 -> [rows, cols/8] uint32, element c = nibble c%8 of word c/8."""
    rows, cols = qmat.shape
    q = qmat.astype(np.uint32).reshape(rows, cols // 8, 8)
    out = np.zeros((rows, cols // 8), np.uint32)
    for j in range(8):
        out |= q[:, :, j] << np.uint32(4 * j)
    return out


def bf16_bits(v) -> np.ndarray:
    return torch.tensor(np.asarray(v, np.float32)).to(torch.bfloat16).view(torch.int16).numpy() \
        .astype(np.uint16)


def const_matrix(rows, cols, q, s, b):
    qm = np.full((rows, cols), q) if np.isscalar(q) else q
    return (pack_nibbles(qm)[None], np.full((1, rows, cols // 64), bf16_bits(s), np.uint16),
            np.full((1, rows, cols // 64), bf16_bits(b), np.uint16))


def one_pair(x_vals, gate, up, down, w=0.5, lib=None):
    H = len(x_vals)
    x = bf16_bits(np.asarray(x_vals, np.float32))[None]
    bank = {"gate": gate, "up": up, "down": down}
    return oracle.switchglu(x, np.zeros((1, 1), np.int32), np.full((1, 1), w, np.float32), bank,
                            1, want_h=True, lib=lib)


def bf16_round_ref(v: np.ndarray) -> np.ndarray:
    """torch's fp32 -> bf16 (round to nearest even) on values exact in fp32."""
    return torch.tensor(np.asarray(v, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


# ------------------------------------------------------------ bf16 rounding ---
def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -133, 3 * 2 ** -134,
                         3.3895313892515355e38, 3.3961e38, 0.7310585786300049]]).astype(np.float32)
    got = np.array([oracle.round_bf16(float(a)) for a in v])
    assert np.array_equal(got, bf16_round_ref(v))


def test_round_bf16_overflow_and_ties():
    assert oracle.round_bf16(1 + 2 ** -8) == 1.0              # tie -> even
    assert oracle.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6  # tie -> even (up)
    assert oracle.round_bf16(255.5 * 2.0 ** 120) == math.inf  # tie at the top -> inf
    assert oracle.round_bf16(255.25 * 2.0 ** 120) == 255 * 2.0 ** 120
    assert oracle.round_bf16(2.0 ** -134) == 0.0              # half the smallest subnormal, tie -> 0
    assert oracle.round_bf16(0.7310585786300049) == 0.73046875


# ------------------------------------------------------------- closed forms ---
def test_closed_form_all_ones():
    m = const_matrix(64, 64, 1, 1.0, 0.0)
    out, h = one_pair([1 / 64] * 64, m, m, m)
    assert np.all(h[0] == 0.73046875)
    assert np.all(out == GOLD["A_all_ones"][0])


def test_closed_form_affine_scale_and_bias():
    gu = const_matrix(64, 64, 3, 0.5, -1.0)
    d = const_matrix(64, 64, 2, 0.25, 0.25)
    out, _ = one_pair([1 / 32] * 64, gu, gu, d)
    assert np.all(out == GOLD["B_affine"][0])


def test_closed_form_pure_bias():
    g = const_matrix(64, 64, 0, 1.0, 0.25)
    u = const_matrix(64, 64, 0, 1.0, 0.5)
    d = const_matrix(64, 64, 0, 1.0, 1 / 64)
    out, h = one_pair([1 / 16] * 64, g, u, d)
    assert np.all(h[0] == 1.4609375)
    assert np.all(out == GOLD["C_pure_bias"][0])


def test_closed_form_identity():
    eye = const_matrix(64, 64, np.eye(64, dtype=np.int64), 1.0, 0.0)
    xs = [2.0, -1.0, 0.5, -3.0, 0.0]
    names = ["x2", "xm1", "x0p5", "xm3", "x0"]
    x = np.zeros(64, np.float32)
    x[:5] = xs
    out, h = one_pair(x, eye, eye, eye, w=1.0)
    for i, n in enumerate(names):
        assert h[0][i] == GOLD["D_identity_h_" + n][0], n
        assert out[0][i] == GOLD["D_identity_h_" + n][0], n
    assert np.all(h[0][5:] == 0.0)


@pytest.mark.parametrize("col", [0, 1, 5, 7, 8, 13, 63, 64, 71, 127])
def test_nibble_and_group_probe(col):
    """A single non-zero code at column `col` of row 0 moves G_0 to 5 * scale(group) * x_col."""
    H = 128
    qm = np.zeros((64, H), np.int64)
    qm[0, col] = 5
    s = np.ones((1, 64, H // 64), np.uint16) * bf16_bits(1.0)
    s[0, :, 1] = bf16_bits(2.0)   # second group scaled by 2
    gate = (pack_nibbles(qm)[None], s, np.zeros((1, 64, H // 64), np.uint16))
    zero = const_matrix(H, 64, 0, 1.0, 0.0)
    x = np.arange(1, H + 1, dtype=np.float32) / 8      # distinct, exact in bf16
    out, h = one_pair(x, gate, gate, zero)
    g = float(bf16_round_ref(np.float32(5 * (1.0 if col < 64 else 2.0) * x[col])))
    expect = bf16_round_ref(np.float32(g * g / (1 + math.exp(-g))))
    assert h[0][0] == expect
    assert np.all(h[0][1:] == 0)


# ---------------------------------------------------------------- union ---
def brute_union(idx, E):
    P = idx.size
    flat = idx.ravel()
    valid = [p for p in range(P) if 0 <= flat[p] < E]
    uniq = sorted(set(int(flat[p]) for p in valid))
    plist, offs = [], [0]
    for e in uniq:
        plist += [p for p in valid if flat[p] == e]
        offs.append(len(plist))
    return uniq, offs, plist + [-1] * (P - len(plist)), P - len(valid)


@pytest.mark.parametrize("seed", range(12))
def test_route_union_brute_force(seed):
    rng = np.random.default_rng(seed)
    T, k, E = int(rng.integers(1, 20)), int(rng.integers(1, 9)), int(rng.integers(1, 300))
    idx = rng.integers(-2, E + 2, size=(T, k)).astype(np.int32)   # duplicates and bad ids
    uniq, offs, plist, u, bad = oracle.route_union(idx, E)
    bu, bo, bp, bbad = brute_union(idx, E)
    assert list(uniq) == bu and list(offs) == bo and list(plist) == bp and bad == bbad
    assert u == len(set(int(e) for e in idx.ravel() if 0 <= e < E))


def test_route_union_extremes():
    T, k, E = 16, 8, 256
    same = np.tile(np.arange(8, dtype=np.int32) * 3, (T, 1))
    uniq, offs, plist, u, _ = oracle.route_union(same, E)
    assert u == k and list(np.diff(offs)) == [T] * k
    disjoint = np.arange(T * k, dtype=np.int32).reshape(T, k)
    uniq, offs, plist, u, _ = oracle.route_union(disjoint, E)
    assert u == T * k and list(plist) == list(range(T * k))


# ------------------------------------------------------- dedup == per pair ---
@pytest.mark.parametrize("cfg", [(2, 2, 16, 256, 128, "softmax"), (5, 4, 8, 128, 192, "uniform"),
                                 (6, 3, 4, 64, 64, "uniform")])
def test_dedup_equals_per_pair_bitwise(cfg):
    T, k, E, H, I, routing = cfg
    L = make_layer(T, k, E, H, I, seed=3, routing=routing)
    out, h = oracle.switchglu(L.x, L.idx, L.w, L.bank, E, want_h=True)
    out2, h2 = oracle.switchglu_union(L.x, L.idx, L.w, L.bank, E, want_h=True)
    assert np.array_equal(out, out2) and np.array_equal(h, h2)


def test_duplicate_expert_in_token_counts_twice():
    L = make_layer(1, 2, 4, 64, 64, seed=5, idx=np.array([[2, 2]], np.int32),
                   w=np.array([[0.25, 0.5]], np.float32))
    single = make_layer(1, 1, 4, 64, 64, seed=5, idx=np.array([[2]], np.int32),
                        w=np.array([[1.0]], np.float32))
    out = oracle.switchglu(L.x, L.idx, L.w, L.bank, 4)
    y = oracle.switchglu(single.x, single.idx, single.w, single.bank, 4)
    assert np.allclose(out, 0.75 * y, rtol=1e-15, atol=0)


# --------------------------------------------------------------- invariants ---
def test_router_weight_scaling_and_zero():
    L = make_layer(3, 4, 12, 128, 64, seed=7)
    base = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E)
    for a in (2.0, 0.5, 0.0):
        got = oracle.switchglu(L.x, L.idx, L.w * np.float32(a), L.bank, L.E)
        assert np.array_equal(got, a * base)


def test_slot_permutation_invariance():
    L = make_layer(3, 4, 12, 128, 64, seed=8)
    base = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E)
    perm = np.array([2, 0, 3, 1])
    got = oracle.switchglu(L.x, L.idx[:, perm], L.w[:, perm], L.bank, L.E)
    assert np.allclose(got, base, rtol=1e-13, atol=1e-12 * np.abs(base).max())


def test_token_independence_and_token_subset():
    L = make_layer(4, 3, 10, 128, 128, seed=9)
    full = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E)
    for t in range(L.T):
        one = oracle.switchglu(L.x[t:t + 1], L.idx[t:t + 1], L.w[t:t + 1], L.bank, L.E)
        assert np.array_equal(one[0], full[t])
    sub = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E, tokens=[2])
    assert np.array_equal(sub[2], full[2]) and np.isnan(sub[0]).all()


def test_invalid_expert_contributes_nothing():
    L = make_layer(2, 3, 6, 64, 64, seed=10, idx=np.array([[1, 7, 2], [-1, 3, 3]], np.int32))
    out = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E)
    w2 = L.w.copy()
    w2[0, 1] = 0
    w2[1, 0] = 0
    idx2 = L.idx.copy()
    idx2[0, 1] = 0
    idx2[1, 0] = 0
    ref = oracle.switchglu(L.x, idx2, w2, L.bank, L.E)
    assert np.array_equal(out, ref)


# ---------------------------------------------------- textbook special case ---
def dense_dequant(q, s, b):
    rows, words = q.shape
    cols = words * 8
    nib = np.stack([(q >> np.uint32(4 * j)) & np.uint32(15) for j in range(8)], axis=-1)
    nib = nib.reshape(rows, cols).astype(np.float64)
    sf = synth.bf16_bits_to_f32(s).astype(np.float64).repeat(64, axis=1)
    bf = synth.bf16_bits_to_f32(b).astype(np.float64).repeat(64, axis=1)
    return sf * nib + bf


@pytest.mark.parametrize("HI", [(128, 64), (256, 192)])
def test_single_expert_is_dense_swiglu(HI):
    H, I = HI
    L = make_layer(1, 1, 1, H, I, seed=11, idx=np.zeros((1, 1), np.int32),
                   w=np.ones((1, 1), np.float32))
    out, h = oracle.switchglu(L.x, L.idx, L.w, L.bank, 1, want_h=True)
    Wg = dense_dequant(L.bank["gate"][0][0], L.bank["gate"][1][0], L.bank["gate"][2][0])
    Wu = dense_dequant(L.bank["up"][0][0], L.bank["up"][1][0], L.bank["up"][2][0])
    Wd = dense_dequant(L.bank["down"][0][0], L.bank["down"][1][0], L.bank["down"][2][0])
    x = synth.bf16_bits_to_f32(L.x[0]).astype(np.float64)
    g = bf16_round_ref(Wg @ x)
    v = bf16_round_ref(Wu @ x)
    href = bf16_round_ref(g * v / (1 + np.exp(-g)))
    # library sums may differ from the oracle's ascending order in the last bits: allow one
    # bf16 step where a value sits on a rounding boundary, and compare y tightly
    ulp = np.abs(href) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(h[0] - href) <= ulp)
    assert np.mean(h[0] == href) > 0.97
    yref = Wd @ h[0]
    assert np.allclose(out[0], yref, rtol=1e-12, atol=1e-12 * np.abs(yref).max())


def test_tiny_layer_runs_and_is_finite():
    L = tiny_layer()
    out = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E)
    assert np.isfinite(out).all() and np.abs(out).max() > 0


# ----------------------------------------------------------- planted mistakes ---
MUTANTS = {
    "nibble_msb_first": ("(word >> (4 * (col % 8)))", "(word >> (4 * (7 - col % 8)))"),
    "bias_dropped": ("return bf16_value(s[g]) * nib + bf16_value(b[g]);",
                     "return bf16_value(s[g]) * nib;"),
    "gate_not_rounded": ("const double g = round_bf16(G), v = round_bf16(U);",
                         "const double g = G, v = round_bf16(U);"),
    "sigmoid_sign": ("std::exp(-g)", "std::exp(g)"),
    "router_weight_dropped": ("acc += static_cast<double>(L.w[p]) * Y[",
                              "acc += Y["),
    "down_transposed": ("Y += L.down.at(e, c, r) * h[r];", "Y += L.down.at(e, r, c) * h[r];"),
    "h_product_unrounded": ("h[r] = round_bf16(g * sigmoid(g) * v);", "h[r] = g * sigmoid(g) * v;"),
    "mxfp4_table_swapped": ("0.0,  0.5,  1.0,  1.5,  2.0,  3.0,  4.0,  6.0,",
                            "0.0,  0.5,  1.0,  2.0,  1.5,  3.0,  4.0,  6.0,"),
    "mxfp4_scale_bias": ("static_cast<int>(v) - 127)", "static_cast<int>(v) - 126)"),
    "router_ascending": ("[row](int a, int b) { return row[a] > row[b]; }",
                         "[row](int a, int b) { return row[a] < row[b]; }"),
    "router_ties_to_higher_id": ("[row](int a, int b) { return row[a] > row[b]; }",
                                 "[row](int a, int b) { return row[a] > row[b] || (row[a] == row[b] && a > b); }"),
    "router_not_renormalised": ("    if (renormalize) {\n      for (int j = 0; j < k; ++j)",
                                "    if (false) {\n      for (int j = 0; j < k; ++j)"),
}

_MUTANT_CHECK = r"""
import sys, numpy as np
sys.path.insert(0, {root!r})
import oracle
from tests import test_oracle_pins as P
lib = oracle.load({so!r})
fails = 0
def run(f):
    global fails
    try:
        f(lib)
    except AssertionError:
        fails += 1
run(P._pin_closed_forms)
run(P._pin_textbook)
run(P._pin_router)
run(P._pin_mxfp4)
print("FAILS", fails)
"""


def _pin_closed_forms(lib):
    m = const_matrix(64, 64, 1, 1.0, 0.0)
    out, _ = one_pair([1 / 64] * 64, m, m, m, lib=lib)
    assert np.all(out == GOLD["A_all_ones"][0])
    gu = const_matrix(64, 64, 3, 0.5, -1.0)
    d = const_matrix(64, 64, 2, 0.25, 0.25)
    out, _ = one_pair([1 / 32] * 64, gu, gu, d, lib=lib)
    assert np.all(out == GOLD["B_affine"][0])
    g = const_matrix(64, 64, 0, 1.0, 0.25)
    u = const_matrix(64, 64, 0, 1.0, 0.5)
    dd = const_matrix(64, 64, 0, 1.0, 1 / 64)
    out, _ = one_pair([1 / 16] * 64, g, u, dd, lib=lib)
    assert np.all(out == GOLD["C_pure_bias"][0])
    eye = const_matrix(64, 64, np.eye(64, dtype=np.int64), 1.0, 0.0)
    x = np.zeros(64, np.float32)
    x[:4] = [2.0, -1.0, 0.5, -3.0]
    out, h = one_pair(x, eye, eye, eye, w=1.0, lib=lib)
    assert h[0][0] == GOLD["D_identity_h_x2"][0] and h[0][3] == GOLD["D_identity_h_xm3"][0]


def _pin_textbook(lib):
    H, I = 128, 64
    L = make_layer(1, 1, 1, H, I, seed=11, idx=np.zeros((1, 1), np.int32),
                   w=np.full((1, 1), 0.75, np.float32))
    qidx = np.zeros((1, 1), np.int32)
    out, h = oracle.switchglu(L.x, qidx, L.w, L.bank, 1, want_h=True, lib=lib)
    Wg = dense_dequant(*[a[0] for a in L.bank["gate"]])
    Wu = dense_dequant(*[a[0] for a in L.bank["up"]])
    Wd = dense_dequant(*[a[0] for a in L.bank["down"]])
    x = synth.bf16_bits_to_f32(L.x[0]).astype(np.float64)
    g = bf16_round_ref(Wg @ x)
    v = bf16_round_ref(Wu @ x)
    href = bf16_round_ref(g * v / (1 + np.exp(-g)))
    assert np.mean(h[0] == href) > 0.97
    yref = 0.75 * (Wd @ href)
    assert np.allclose(out[0], yref, rtol=0, atol=1e-3 * np.abs(yref).max())


def _pin_router(lib):
    # equal logits: the k lowest ids, weights 1/k renormalised, 1/E otherwise
    E, k = 12, 5
    idx, w = oracle.router_topk(np.full((2, E), 0.75, np.float32), k, True, lib=lib)
    assert np.array_equal(idx, np.tile(np.arange(k), (2, 1)))
    assert np.allclose(w, 1.0 / k, rtol=1e-15, atol=0)
    _, w = oracle.router_topk(np.full((1, E), -2.5, np.float32), k, False, lib=lib)
    assert np.allclose(w, 1.0 / E, rtol=1e-15, atol=0)
    # logits ln(i + 1): softmax_i = (i + 1) / sum; the top k are the last k ids
    E, k = 40, 6
    lg = np.log(np.arange(1, E + 1, dtype=np.float64)).astype(np.float32)[None]
    idx, w = oracle.router_topk(lg, k, True, lib=lib)
    top = np.arange(E - 1, E - 1 - k, -1)
    assert np.array_equal(idx[0], top)
    assert np.allclose(w[0], (top + 1) / np.sum(top + 1), rtol=1e-6, atol=0)
    _, w = oracle.router_topk(lg, k, False, lib=lib)
    assert np.allclose(w[0], (top + 1) / (E * (E + 1) / 2), rtol=1e-6, atol=0)
    # one id ahead of an equal one: a tie resolves to the lower id
    lg = np.zeros((1, 8), np.float32)
    lg[0, [2, 6]] = 1.0
    idx, _ = oracle.router_topk(lg, 3, True, lib=lib)
    assert list(idx[0]) == [2, 6, 0]


def _e2m1_codes(vals: np.ndarray) -> np.ndarray:
    """e2m1 codes of values the format holds exactly, encoded by ml_dtypes."""
    import ml_dtypes
    return np.asarray(vals, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15


def _shared_banks(rng, E, H, I, e8, s, b):
    """Random weights from {0, +-0.5, +-1, +-1.5, +-2, +-3} * 2^(e8 - 127), held
    exactly both as mxfp4 (scale e8) and as affine (scale s, bias b)."""
    vals = np.array([0, 0.5, -0.5, 1, -1, 1.5, -1.5, 2, -2, 3, -3])
    mx, af = {}, {}
    for name, rows, cols in (("gate", I, H), ("up", I, H), ("down", H, I)):
        v = rng.choice(vals, size=(E, rows, cols))
        scale = 2.0 ** (e8 - 127)
        mx[name] = (np.stack([pack_nibbles(_e2m1_codes(v[e])) for e in range(E)]),
                    np.full((E, rows, cols // 32), e8, np.uint8))
        q = np.rint((v * scale - b) / s).astype(np.int64)
        assert q.min() >= 0 and q.max() <= 15 and np.all(q * s + b == v * scale)
        af[name] = (np.stack([pack_nibbles(q[e]) for e in range(E)]),
                    np.full((E, rows, cols // 64), bf16_bits(s), np.uint16),
                    np.full((E, rows, cols // 64), bf16_bits(b), np.uint16))
    return mx, af


def _pin_mxfp4(lib):
    import ml_dtypes
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for e8 in (100, 120, 126, 127, 128, 131, 150):
        sc = float(np.array([e8], np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)[0])
        got = np.array([oracle.mxfp4_value(c, e8, lib=lib) for c in range(16)])
        assert np.array_equal(got, ref * sc)
    rng = np.random.default_rng(23)
    T, k, E, H, I = 3, 2, 4, 128, 64
    x = bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    idx = np.array([[0, 3], [2, 2], [1, 0]], np.int32)
    w = np.array([[0.25, 0.75], [0.5, 0.5], [1.0, -0.5]], np.float32)
    for e8, s, b in ((127, 0.5, -3.0), (128, 1.0, -6.0), (125, 0.125, -0.75)):
        mx, af = _shared_banks(rng, E, H, I, e8, s, b)
        out_mx = oracle.switchglu_mxfp4(x, idx, w, mx, E, lib=lib)
        out_af = oracle.switchglu(x, idx, w, af, E, lib=lib)
        assert np.array_equal(out_mx, out_af)


def test_mxfp4_pins():
    _pin_mxfp4(oracle.load())


def test_mxfp4_single_expert_is_dense_swiglu():
    """E=1, k=1 with random codes and scales: the mxfp4 layer equals a dense SwiGLU
    of the matrices decoded by ml_dtypes (numpy matmul)."""
    import ml_dtypes
    rng = np.random.default_rng(29)
    H, I = 128, 64
    bank, dense = {}, {}
    for name, rows, cols in (("gate", I, H), ("up", I, H), ("down", H, I)):
        c = rng.integers(0, 16, size=(rows, cols)).astype(np.uint8)
        e8 = rng.integers(118, 124, size=(rows, cols // 32)).astype(np.uint8)
        bank[name] = (pack_nibbles(c)[None], e8[None])
        vals = c.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        dense[name] = vals * e8.view(ml_dtypes.float8_e8m0fnu).astype(np.float64).repeat(32, axis=1)
    xf = rng.standard_normal(H).astype(np.float32)
    x = bf16_bits(xf)[None]
    out, h = oracle.switchglu_mxfp4(x, np.zeros((1, 1), np.int32), np.full((1, 1), 0.75, np.float32),
                                    bank, 1, want_h=True)
    xd = synth.bf16_bits_to_f32(x[0]).astype(np.float64)
    g = bf16_round_ref(dense["gate"] @ xd)
    v = bf16_round_ref(dense["up"] @ xd)
    href = bf16_round_ref(g * v / (1 + np.exp(-g)))
    assert np.mean(h[0] == href) > 0.97
    yref = 0.75 * (dense["down"] @ href)
    assert np.allclose(out[0], yref, rtol=0, atol=1e-3 * np.abs(yref).max())


def test_router_pins():
    _pin_router(oracle.load())


def test_router_against_library_routines():
    """k = E gives the full softmax (scipy), sorted descending; the selection of
    distinct logits equals torch.topk's; adding an exactly representable constant
    changes nothing."""
    from scipy.special import softmax
    rng = np.random.default_rng(41)
    for T, E, k in [(3, 16, 16), (5, 288, 8), (2, 1024, 32), (4, 7, 3)]:
        lg = (rng.permutation(E * T).reshape(T, E) / 64.0 - 4.0).astype(np.float32)  # distinct
        idx, w = oracle.router_topk(lg, k, renormalize=(k != E))
        ti = torch.topk(torch.from_numpy(lg).double(), k, dim=1, sorted=True).indices.numpy()
        assert np.array_equal(idx, ti)
        if k == E:
            ref = softmax(lg.astype(np.float64), axis=1)
            assert np.allclose(w, np.take_along_axis(ref, idx, axis=1), rtol=1e-12, atol=0)
        idx2, w2 = oracle.router_topk(lg + np.float32(2.0), k, renormalize=(k != E))
        assert np.array_equal(idx, idx2) and np.allclose(w, w2, rtol=1e-12, atol=0)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.cpp")).read()
    assert old in src, "mutation site vanished: update the mutant"
    mpath = tmp_path / "oracle_mut.cpp"
    mpath.write_text(src.replace(old, new))
    so = str(tmp_path / "liboracle_mut.so")
    oracle.build(str(mpath), so)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _MUTANT_CHECK.format(root=root, so=so)],
                       capture_output=True, text=True, timeout=300)
    assert "FAILS" in r.stdout, r.stderr[-2000:]
    assert int(r.stdout.split("FAILS")[1].split()[0]) >= 1, f"mutant {name} passed every pin"


def test_unmutated_oracle_passes_mutant_pins():
    lib = oracle.load()
    _pin_closed_forms(lib)
    _pin_textbook(lib)
    _pin_router(lib)
    _pin_mxfp4(lib)
