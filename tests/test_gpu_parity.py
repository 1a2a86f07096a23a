"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Integer outputs (route-union arrays) must match bit for bit; the bf16 layer
output must be within rel-L2 5e-3 and max-abs/rms(ref) 3e-2 of the oracle on the
same seeded inputs.  Shapes span several row blocks and a ragged tail; the
full-size layers are the shapes the pages measure (GLM-5.3-Flash-shaped
E=288 top-8 4096/2048; the E=256 verify pair and verify windows).
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_gather_b200 as qeg
import synth
from tests.gpu_util import assert_parity, bf16_to_f64, to_dev_bank, to_dev_inputs
from tests.layers import make_layer, tiny_layer

pytestmark = pytest.mark.gpu


def bf16_round(v: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 (nearest even) through the oracle's own rounding, elementwise."""
    return np.vectorize(oracle.round_bf16)(v)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """One bf16 step at |v| (8 significant bits)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def dense_dequant(q, s, b):
    """Dense fp64 rows of one packed matrix: s * q + b per group of 64 columns."""
    rows, words = q.shape
    nib = np.stack([(q >> np.uint32(4 * j)) & np.uint32(15) for j in range(8)], axis=-1)
    nib = nib.reshape(rows, words * 8).astype(np.float64)
    sf = synth.bf16_bits_to_f32(s).astype(np.float64).repeat(64, axis=1)
    bf = synth.bf16_bits_to_f32(b).astype(np.float64).repeat(64, axis=1)
    return sf * nib + bf


def run_forward(L, ws=False):
    bank = to_dev_bank(L)
    x, idx, w = to_dev_inputs(L)
    if ws:
        work = qeg.moe_workspace(L.T, L.k, L.E, L.H, L.I)
        out = qeg.moe_switchglu_forward_ws(x, idx, w, bank, work)
    else:
        out = qeg.moe_switchglu_forward(x, idx, w, bank)
    torch.cuda.synchronize()
    return out, (bank, x, idx, w)


def check_layer(L, what, tokens=None):
    out, _ = run_forward(L)
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    ref = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E, tokens=tokens)
    got = bf16_to_f64(out)
    if tokens is not None:
        got, ref = got[tokens], ref[tokens]
    assert_parity(got, ref, what)
    return out


# ------------------------------------------------------------- route-union ---
@pytest.mark.parametrize("seed", range(8))
def test_route_union_bit_exact_random(seed):
    rng = np.random.default_rng(100 + seed)
    T, k = int(rng.integers(1, 40)), int(rng.integers(1, 9))
    E = int(rng.integers(1, 1025))
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    uq, of, pl, nu = qeg.moe_route_union(torch.from_numpy(idx).cuda(), E)
    u_ref, o_ref, p_ref, n_ref, _ = oracle.route_union(idx, E)
    n = int(nu.item())
    assert n == n_ref
    assert np.array_equal(uq.cpu().numpy()[:n], u_ref)
    assert np.array_equal(of.cpu().numpy()[:n + 1], o_ref)
    assert np.array_equal(pl.cpu().numpy(), p_ref)
    assert qeg.moe_read_device_status() == qeg.MOE_OK


@pytest.mark.parametrize("T,k,E", [(1, 8, 288), (4, 8, 288), (16, 8, 256), (512, 8, 256),
                                   (2048, 8, 256), (8192, 8, 1024), (3, 1, 1)])
def test_route_union_bit_exact_sizes(T, k, E):
    idx, _ = synth.route_uniform(T, E, k, seed=T * 7 + E) if k <= E else (None, None)
    if idx is None:
        idx = np.zeros((T, k), np.int32)
    uq, of, pl, nu = qeg.moe_route_union(torch.from_numpy(idx).cuda(), E)
    u_ref, o_ref, p_ref, n_ref, _ = oracle.route_union(idx, E)
    n = int(nu.item())
    assert n == n_ref and np.array_equal(uq.cpu().numpy()[:n], u_ref)
    assert np.array_equal(of.cpu().numpy()[:n + 1], o_ref)
    assert np.array_equal(pl.cpu().numpy(), p_ref)


def test_route_union_extremes_and_invalid_ids():
    T, k, E = 16, 8, 256
    for idx in (np.tile(np.arange(8, dtype=np.int32) * 5, (T, 1)),
                np.arange(T * k, dtype=np.int32).reshape(T, k)):
        uq, of, pl, nu = qeg.moe_route_union(torch.from_numpy(idx).cuda(), E)
        u_ref, o_ref, p_ref, n_ref, _ = oracle.route_union(idx, E)
        assert int(nu.item()) == n_ref and np.array_equal(pl.cpu().numpy(), p_ref)
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    bad = np.array([[3, 300, 3], [-1, 7, 255]], np.int32)
    uq, of, pl, nu = qeg.moe_route_union(torch.from_numpy(bad).cuda(), E)
    u_ref, o_ref, p_ref, n_ref, nbad = oracle.route_union(bad, E)
    assert nbad == 2 and int(nu.item()) == n_ref and np.array_equal(pl.cpu().numpy(), p_ref)
    assert qeg.moe_read_device_status() == qeg.MOE_ERR_DEVICE_INDEX
    assert qeg.moe_read_device_status() == qeg.MOE_OK  # cleared by the read


# ----------------------------------------------------------------- forward ---
def test_tiny_layer():
    check_layer(tiny_layer(), "tiny E=16 top-2 256/128 T=2")


@pytest.mark.parametrize("cfg", [
    # T, k, E, H, I, routing
    (7, 6, 40, 512, 384, "uniform"),     # ragged: several row blocks, odd T
    (1, 8, 64, 256, 192, "uniform"),
    (5, 3, 8, 1024, 512, "uniform"),     # heavy sharing: ~2 tokens per expert
    (16, 8, 256, 512, 256, "markov"),
    (3, 2, 4, 4096, 128, "uniform"),     # full hidden width, small inter
    (9, 4, 30, 192, 1088, "uniform"),    # inter > 1024 (two chunk-warps), ragged
])
def test_forward_small_shapes(cfg):
    T, k, E, H, I, routing = cfg
    L = make_layer(T, k, E, H, I, seed=sum(cfg[:5]), routing=routing)
    check_layer(L, f"T={T} k={k} E={E} H={H} I={I}")


def test_forward_ws_variant_and_union_export():
    L = make_layer(6, 4, 24, 256, 256, seed=21)
    out, (bank, x, idx, w) = run_forward(L)
    work = qeg.moe_workspace(L.T, L.k, L.E, L.H, L.I)
    out2 = qeg.moe_switchglu_forward_ws(x, idx, w, bank, work)
    torch.cuda.synchronize()
    lay = qeg.moe_workspace_layout(L.T, L.k, L.E, L.H, L.I)
    assert not work[lay["barrier"]:lay["num_unique"]].any()  # progress counters back to zero
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    wsn = work.cpu().numpy()
    u = int(wsn[lay["num_unique"]:lay["num_unique"] + 4].view(np.int32)[0])
    u_ref, o_ref, p_ref, n_ref, _ = oracle.route_union(L.idx, L.E)
    assert u == n_ref
    assert np.array_equal(wsn[lay["unique"]:lay["unique"] + 4 * u].view(np.int32), u_ref)
    P = L.T * L.k
    assert np.array_equal(wsn[lay["pair_list"]:lay["pair_list"] + 4 * P].view(np.int32), p_ref)
    # h in pair_list order vs the oracle's per-pair h.  The kernel's G and U differ from
    # the oracle's fp64 sums by rounding (fp32 sums, activations in 16-bit block fixed
    # point), so where G or U sits near a bf16 rounding boundary g or v may be one bf16
    # step off; h may then move by |dh/dg| ulp(g) + |dh/dv| ulp(v), plus its own step.
    _, h_ref = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E, want_h=True)
    h = torch.from_numpy(wsn[lay["h"]:lay["h"] + 2 * P * L.I].view(np.int16).copy()) \
        .view(torch.bfloat16).float().numpy().reshape(P, L.I).astype(np.float64)
    n_valid = o_ref[-1]
    h_ref_sorted = h_ref[p_ref[:n_valid]]
    x64 = synth.bf16_bits_to_f32(L.x).astype(np.float64)
    G = np.empty((n_valid, L.I))
    U = np.empty((n_valid, L.I))
    for i, p in enumerate(p_ref[:n_valid]):
        t, e = p // L.k, L.idx[p // L.k, p % L.k]
        G[i] = dense_dequant(*[a[e] for a in L.bank["gate"]]) @ x64[t]
        U[i] = dense_dequant(*[a[e] for a in L.bank["up"]]) @ x64[t]
    g, v = bf16_round(G), bf16_round(U)
    sig = 1.0 / (1.0 + np.exp(-g))
    dh_dg = np.abs(v * (sig + g * sig * (1.0 - sig)))
    dh_dv = np.abs(g * sig)
    abs_g = 1e-4 * np.sqrt(np.mean(G ** 2))  # absolute slack for G near zero
    abs_v = 1e-4 * np.sqrt(np.mean(U ** 2))
    tol = (dh_dg * (bf16_ulp(g) + abs_g) + dh_dv * (bf16_ulp(v) + abs_v)
           + bf16_ulp(h_ref_sorted))
    err = np.abs(h[:n_valid] - h_ref_sorted)
    assert np.all(err <= 1.5 * tol), float(np.max(err / np.maximum(tol, 1e-300)))
    assert np.mean(h[:n_valid] == h_ref_sorted) > 0.97


def test_deterministic_bitwise():
    L = make_layer(8, 8, 64, 1024, 512, seed=31, routing="markov", p=0.5)
    a, _ = run_forward(L)
    b, _ = run_forward(L)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_token_independence():
    L = make_layer(4, 8, 32, 512, 256, seed=41, routing="markov", p=0.6)
    full, _ = run_forward(L)
    for t in range(L.T):
        one = make_layer(1, 8, 32, 512, 256, seed=41, idx=L.idx[t:t + 1], w=L.w[t:t + 1])
        one.x = L.x[t:t + 1]
        one.bank = L.bank
        o, _ = run_forward(one)
        assert_parity(bf16_to_f64(o)[0:1], bf16_to_f64(full)[t:t + 1], f"token {t}")


def test_duplicate_experts_zero_weights_and_invalid_ids():
    E = 12
    idx = np.array([[2, 2, 5], [7, 13, 1], [-4, 3, 3], [0, 1, 2]], np.int32)
    w = np.array([[0.5, 0.25, 0.25], [0.2, 0.3, 0.5], [1.0, 0.5, 0.5], [0, 0, 0]], np.float32)
    L = make_layer(4, 3, E, 256, 128, seed=51, idx=idx, w=w)
    out, _ = run_forward(L)
    assert qeg.moe_read_device_status() == qeg.MOE_ERR_DEVICE_INDEX
    ref = oracle.switchglu(L.x, L.idx, L.w, L.bank, E)
    got = bf16_to_f64(out)
    assert not np.any(got[3])  # zero router weights -> zero row
    assert_parity(got, ref, "duplicates / invalid ids")


def test_all_invalid_gives_zero_rows():
    idx = np.full((3, 4), 99, np.int32)
    L = make_layer(3, 4, 8, 128, 64, seed=52, idx=idx)
    out, _ = run_forward(L)
    assert qeg.moe_read_device_status() == qeg.MOE_ERR_DEVICE_INDEX
    assert not torch.any(out.float() != 0)


def test_all_identical_and_disjoint_routing():
    T, k, E, H, I = 16, 8, 256, 512, 256
    same = np.tile(np.arange(8, dtype=np.int32) * 9, (T, 1))
    check_layer(make_layer(T, k, E, H, I, seed=61, idx=same), "all-identical routing")
    disjoint = np.arange(T * k, dtype=np.int32).reshape(T, k)
    check_layer(make_layer(T, k, E, H, I, seed=62, idx=disjoint), "disjoint routing")


# ---------------------------------------------------------- full-size layers ---
@pytest.mark.parametrize("T", [1, 4])
def test_glm_flash_layer(T):
    """E=288, top-8, hidden 4096, intermediate 2048, uniform routing (the moe_bench.py layer)."""
    L = make_layer(T, 8, 288, 4096, 2048, seed=2000 + T, routing="uniform")
    check_layer(L, f"GLM-5.3-Flash-shaped T={T}")


@pytest.mark.parametrize("p", [0.03, 0.34, 0.52])
def test_verify_pair_layer(p):
    idx, w = synth.route_verify_pair(256, 8, p, seed=3000 + int(p * 100))
    L = make_layer(2, 8, 256, 4096, 2048, seed=3000 + int(p * 100), idx=idx, w=w)
    check_layer(L, f"verify pair p={p}")


@pytest.mark.parametrize("T", [3, 16])
def test_verify_window_layer(T):
    L = make_layer(T, 8, 256, 4096, 2048, seed=4000 + T, routing="markov", p=0.40)
    check_layer(L, f"verify window T={T}")


# ------------------------------------------------------------ generator twin ---
def test_device_generator_matches_host():
    E, rows, cols, seed = 5, 64, 512, 77
    q = torch.zeros((E, rows, cols // 8), dtype=torch.int32, device="cuda")
    s = torch.zeros((E, rows, cols // 64), dtype=torch.int16, device="cuda")
    b = torch.zeros_like(s)
    synth.fill_bank_device(q, s, b, rows, cols, seed, synth.MATRIX_UP)
    torch.cuda.synchronize()
    qh, sh, bh = synth.fill_bank_host(E, rows, cols, seed, synth.MATRIX_UP)
    assert np.array_equal(q.cpu().numpy().view(np.uint32), qh)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), sh)
    assert np.array_equal(b.cpu().numpy().view(np.uint16), bh)


# ------------------------------------------------------------ argument errors ---
def test_rejected_arguments_launch_nothing():
    L = make_layer(2, 2, 4, 128, 64, seed=71)
    bank = to_dev_bank(L)
    x, idx, w = to_dev_inputs(L)
    # misaligned activation pointer (2 bytes into a real allocation)
    xbig = torch.zeros(2 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    xmis = xbig[1:1 + 2 * 128].view(2, 128)
    assert qeg.moe_switchglu_forward(xmis, idx, w, bank, check=False) is not None
    st = qeg._lib.moe_switchglu_forward(xmis.data_ptr(), idx.data_ptr(), w.data_ptr(),
                                        *bank.ptrs(), 2, 2, 4, 128, 64,
                                        torch.empty(2, 128, dtype=torch.bfloat16,
                                                    device="cuda").data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)
    assert st == qeg.MOE_ERR_UNSUPPORTED
    # workspace too small
    work = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(qeg.MoeError) as ei:
        qeg.moe_switchglu_forward_ws(x, idx, w, bank, work)
    assert ei.value.status == qeg.MOE_ERR_WORKSPACE
    # hidden not a multiple of 64 is an invalid shape, rejected before any launch
    st = qeg._lib.moe_switchglu_forward(x.data_ptr(), idx.data_ptr(), w.data_ptr(), *bank.ptrs(),
                                        2, 2, 4, 96, 64, x.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)
    assert st == qeg.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK


def test_library_workspace_reused_across_shapes():
    """The library-owned workspace serves calls of different shapes in any order: its
    progress counters must stay zero between calls whatever shape came before."""
    shapes = [(16, 8, 64, 1024, 512), (1, 2, 8, 256, 128), (9, 4, 30, 512, 1088),
              (2, 8, 64, 256, 192), (16, 8, 64, 1024, 512)]
    for i, (T, k, E, H, I) in enumerate(shapes):
        L = make_layer(T, k, E, H, I, seed=900 + i, routing="uniform")
        check_layer(L, f"reuse #{i} T={T} k={k} E={E} H={H} I={I}")


# ----------------------------------------------------- large windows (grouped) ---
def test_grouped_path_selected_for_large_windows():
    assert qeg.moe_select_path(160, 8, 64, 512, 256) == 2
    assert qeg.moe_select_path(512, 8, 256, 4096, 2048) == 2
    assert qeg.moe_select_path(2048, 8, 256, 4096, 2048) == 2
    assert qeg.moe_select_path(512, 8, 256, 6144, 2048) == 2
    assert qeg.moe_select_path(160, 8, 64, 512, 192) == 0  # weight rows not a multiple of 128


@pytest.mark.parametrize("cfg", [
    # T, k, E, H, I: several experts with more than 16 pairs, ragged N tiles
    (160, 8, 64, 512, 256),
    (130, 8, 16, 256, 384),
    (130, 8, 16, 6144, 256),  # hidden 6144 (GLM-5.2's width)
    (130, 8, 8, 8192, 128),   # the widest hidden the library takes
])
def test_grouped_small(cfg):
    T, k, E, H, I = cfg
    L = make_layer(T, k, E, H, I, seed=700 + T, routing="uniform")
    check_layer(L, f"grouped T={T} E={E} H={H} I={I}")


def test_grouped_hot_expert_over_256_pairs():
    """Expert 3 in every token: one expert with 300 pairs (two N tiles)."""
    T, k, E, H, I = 300, 4, 32, 256, 256
    rng = np.random.default_rng(9)
    idx = np.stack([np.concatenate([[3], rng.choice([e for e in range(E) if e != 3], k - 1,
                                                    replace=False)]) for _ in range(T)])
    L = make_layer(T, k, E, H, I, seed=91, idx=idx.astype(np.int32))
    check_layer(L, "grouped, one expert with 300 pairs")


def test_grouped_invalid_ids_and_zero_rows():
    T, k, E, H, I = 140, 8, 40, 256, 128
    L = make_layer(T, k, E, H, I, seed=93, routing="uniform")
    L.idx[5, :] = 77      # every pair of token 5 invalid -> zero row
    L.idx[9, 3] = -1
    out, _ = run_forward(L)
    assert qeg.moe_read_device_status() == qeg.MOE_ERR_DEVICE_INDEX
    ref = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E)
    got = bf16_to_f64(out)
    assert not np.any(got[5])
    assert_parity(got, ref, "grouped with invalid ids")


@pytest.mark.parametrize("T,n_check", [(512, 48), (2048, 32)])
def test_grouped_large_window(T, n_check):
    """The large-window configuration: E=256, top-8, 4096/2048, uniform routing; the
    oracle checks a seeded sample of tokens."""
    L = make_layer(T, 8, 256, 4096, 2048, seed=5000 + T, routing="uniform", draw_all=False)
    tokens = sorted(np.random.default_rng(T).choice(T, n_check, replace=False).tolist())
    check_layer(L, f"large window T={T}", tokens=tokens)


# ------------------------------------------------------------- router step ---
# Weights: exp in fp32 (CUDA expf, at most 2 ulp) and fp32 sums of at most 1024 terms
# (32 per lane, then a 5-level butterfly) against fp64: relative error below ~40 ulp
# of fp32 (2.4e-6); the test allows 2e-5.  The picks compare the fp32 logits as given
# on both sides, so they are compared bit for bit.
ROUTER_RTOL = 2e-5


@pytest.mark.parametrize("T,E,k,renorm,ties", [
    (1, 288, 8, True, False), (4, 288, 8, True, False), (16, 256, 8, True, False),
    (2, 16, 2, True, False), (64, 1024, 32, True, False), (33, 1, 1, True, False),
    (7, 288, 8, False, False), (5, 1000, 32, False, False), (300, 64, 8, True, True),
    (4096, 256, 8, True, False), (9, 32, 32, True, True),
])
def test_router_topk_matches_oracle(T, E, k, renorm, ties):
    rng = np.random.default_rng(1000 + T * 7 + E + k)
    lg = rng.standard_normal((T, E))
    if ties:  # many equal logits: the lower expert id must come first
        lg = np.round(lg * 2) / 2
    lg = lg.astype(np.float32)
    idx, w = qeg.moe_router_topk(torch.from_numpy(lg).cuda(), k, renormalize=renorm)
    torch.cuda.synchronize()
    ridx, rw = oracle.router_topk(lg, k, renormalize=renorm)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy().astype(np.float64), rw, rtol=ROUTER_RTOL, atol=0)


def test_router_feeds_the_layer():
    """Logits -> router -> layer on the device, against the oracle's router and layer."""
    L = tiny_layer()
    rng = np.random.default_rng(77)
    lg = rng.standard_normal((L.T, L.E)).astype(np.float32)
    bank = to_dev_bank(L)
    x, _, _ = to_dev_inputs(L)
    idx, w = qeg.moe_router_topk(torch.from_numpy(lg).cuda(), L.k)
    out = qeg.moe_switchglu_forward(x, idx, w, bank)
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    ridx, rw = oracle.router_topk(lg, L.k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    ref = oracle.switchglu(L.x, ridx, rw.astype(np.float32), L.bank, L.E)
    assert_parity(bf16_to_f64(out), ref, "router -> layer")
