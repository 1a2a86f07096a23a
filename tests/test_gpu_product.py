"""Parity of the product configurations the bench and the path selection reach.

* The persistent small-window kernel at full width (hidden 4096, inter 2048) on windows
  of 256 to 1024 pairs, where its shared-memory tables are largest and its ring is
  shallowest, and with experts shared by many pairs (segments of several pairs each).
* Layers issued back to back on one stream with no host synchronisation, and the same
  sequence captured in a CUDA graph and replayed: every layer's output is kept and
  compared with the oracle (the chained mode of "gather_qmm at M=1 streams 4-bit expert
  weights at ~half the bandwidth of M=4", mlx issue 4509, "Numbers": 42 layers chained
  without intermediate sync).
* Activations with outlier channels, against the block fixed-point representation the
  small-window kernel holds them in.
* Every token of the T=512 large window (grouped tensor-core path).
* A bounded wait that runs out: the call reports MOE_ERR_TIMEOUT and returns, and the
  next call is correct again.
* The router step fused into the layer (moe_switchglu_forward_routed): the same picks,
  weights and output, bit for bit, as the router kernel followed by the layer, on the
  persistent path and on the grouped path, and the oracle's router and layer.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_gather_b200 as qeg
import synth
from tests.gpu_util import (assert_parity, bf16_tensor, bf16_to_f64, dev_bank_drawn,
                            to_dev_bank, to_dev_inputs)
from tests.layers import draw_bank, make_layer

pytestmark = pytest.mark.gpu

H, I = 4096, 2048


def sample_tokens(T, n, seed):
    return sorted(np.random.default_rng(seed).choice(T, min(n, T), replace=False).tolist())


def check_sampled(x_bits, idx, w, bank_dev, E, seed, tokens, what):
    """Run the layer on the device bank, compare `tokens` with the oracle on host draws of
    just the experts those tokens use."""
    out = qeg.moe_switchglu_forward(bf16_tensor(x_bits), torch.from_numpy(idx).cuda(),
                                    torch.from_numpy(w).cuda(), bank_dev)
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    used = sorted(set(int(e) for e in idx[tokens].ravel()))
    hb = draw_bank(E, H, I, seed, used)
    ref = oracle.switchglu(x_bits, idx, w, hb, E, tokens=tokens)
    assert_parity(bf16_to_f64(out)[tokens], ref[tokens], what)
    return out


@pytest.mark.parametrize("T,k,routing", [(32, 8, "uniform"), (64, 8, "markov"),
                                         (128, 8, "uniform"), (1024, 1, "uniform")])
def test_persistent_kernel_large_windows_full_width(T, k, routing):
    """Windows of 256-1024 pairs at 4096/2048 go to the persistent kernel (path 1)."""
    E, seed = 256, 6000 + T * k
    assert qeg.moe_select_path(T, k, E, H, I) == 1
    bank = dev_bank_drawn(E, H, I, seed)
    if routing == "markov":
        idx, w = synth.route_markov(T, E, k, 0.4, seed)
    else:
        idx, w = synth.route_uniform(T, E, k, seed)
    x = synth.x_bf16(T, H, seed)
    tokens = sample_tokens(T, 12, seed)
    check_sampled(x, idx, w, bank, E, seed, tokens, f"persistent kernel T={T} k={k}")


def test_persistent_kernel_hot_experts_full_width():
    """Every token routes to experts 0..3, plus 4 of its own: four experts with 16 pairs
    each (several segments per expert) next to experts with one pair."""
    T, k, E, seed = 16, 8, 256, 6100
    rng = np.random.default_rng(seed)
    idx = np.stack([np.concatenate([[0, 1, 2, 3], rng.choice(np.arange(4, E), 4,
                                                             replace=False)])
                    for _ in range(T)]).astype(np.int32)
    w = synth.route_uniform(T, E, k, seed)[1]
    bank = dev_bank_drawn(E, H, I, seed)
    check_sampled(synth.x_bf16(T, H, seed), idx, w, bank, E, seed, list(range(T)),
                  "hot experts T=16")


# ------------------------------------------------------------- chained layers ---
def _chain(E=64, seed=6200):
    """A chain of layers on one bank: window sizes, routings and router weights differ per
    layer (as in a decode step, each layer its own routing)."""
    Ts = [1, 4, 2, 16, 3, 1, 8, 5, 4, 1]
    layers = []
    for l, T in enumerate(Ts):
        if l % 2:
            idx, w = synth.route_markov(T, E, 8, 0.4, seed + l)
        else:
            idx, w = synth.route_uniform(T, E, 8, seed + l)
        layers.append((synth.x_bf16(T, H, seed + 50 + l), idx, w))
    return Ts, layers


def test_chained_layers_back_to_back_and_graph_replay():
    """Ten layers on one stream with no host synchronisation between them (each launch may
    start under the previous one's tail), then the same ten captured in a CUDA graph and
    replayed twice.  Every output is kept and compared with the oracle, and the replays
    must reproduce the eager outputs bit for bit.  Both the caller-owned workspace (one
    shared by all layers, as the bench does) and the library-owned one are covered."""
    E, seed = 64, 6200
    bank = dev_bank_drawn(E, H, I, seed)
    hb = draw_bank(E, H, I, seed)
    Ts, layers = _chain(E, seed)
    dev = [(bf16_tensor(x), torch.from_numpy(i).cuda(), torch.from_numpy(w).cuda())
           for x, i, w in layers]
    refs = [oracle.switchglu(x, i, w, hb, E) for x, i, w in layers]
    ws = qeg.moe_workspace(max(Ts), 8, E, H, I)
    for owned in (False, True):
        outs = [torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
                for T in Ts]

        def issue():
            for (x, i, w), o in zip(dev, outs):
                if owned:
                    qeg.moe_switchglu_forward(x, i, w, bank, out=o)
                else:
                    qeg.moe_switchglu_forward_ws(x, i, w, bank, ws, out=o)

        issue()  # eager, back to back
        torch.cuda.synchronize()
        assert qeg.moe_read_device_status() == qeg.MOE_OK
        eager = [o.clone() for o in outs]
        for l, (o, ref) in enumerate(zip(eager, refs)):
            assert_parity(bf16_to_f64(o), ref, f"chained layer {l} (T={Ts[l]}, owned={owned})")
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            issue()
        for o in outs:
            o.fill_(float("nan"))
        for rep in range(2):
            g.replay()
            torch.cuda.synchronize()
            assert qeg.moe_read_device_status() == qeg.MOE_OK
            for l, (o, e) in enumerate(zip(outs, eager)):
                assert torch.equal(o.view(torch.int16), e.view(torch.int16)), \
                    f"graph replay {rep}, layer {l}: differs from the eager output"
            for o in outs:
                o.fill_(float("nan"))
        del g
    lay = qeg.moe_workspace_layout(max(Ts), 8, E, H, I)
    assert not ws[lay["barrier"]:lay["num_unique"]].any()  # counters back to zero


# --------------------------------------------------------- outlier activations ---
def test_outlier_activation_channels():
    """x with a few channels scaled by 256-1024 (outlier features of decoder activations)
    and one 32-column chunk whose values span more than 2^12 in magnitude.  The kernel
    holds x and h in 16-bit block fixed point per 32 columns; values far below their
    chunk's largest lose low bits, which the output tolerance must absorb."""
    T, k, E, seed = 4, 8, 64, 6300
    L = make_layer(T, k, E, H, I, seed=seed, routing="uniform")
    xf = synth.bf16_bits_to_f32(L.x).astype(np.float32)
    for ch, f in ((5, 512.0), (1000, 1024.0), (2047, 256.0), (3333, 768.0), (4095, 300.0)):
        xf[:, ch] *= f
    xf[:, 320] = 4096.0 * np.sign(xf[:, 320] + 1e-3)   # chunk 10: +-4096 next to N(0,1)
    xf[:, 321] = 2.0 ** -6                                # and 2^-18 of it
    L.x = synth.f32_to_bf16_bits(xf)
    ref = oracle.switchglu(L.x, L.idx, L.w, L.bank, E)
    bank = to_dev_bank(L)
    x, idx, w = to_dev_inputs(L)
    out = qeg.moe_switchglu_forward(x, idx, w, bank)
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    assert_parity(bf16_to_f64(out), ref, "outlier activation channels")
    got = bf16_to_f64(out)  # and token by token
    for t in range(T):
        assert_parity(got[t:t + 1], ref[t:t + 1], f"outliers, token {t}")


# ------------------------------------------------------------ every token T=512 ---
def test_grouped_large_window_every_token():
    """T=512, E=256, top-8, 4096/2048, uniform routing: every token against the oracle."""
    T = 512
    L = make_layer(T, 8, 256, H, I, seed=5000 + T, routing="uniform")
    out = qeg.moe_switchglu_forward(*to_dev_inputs(L), to_dev_bank(L))
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    ref = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E)
    got = bf16_to_f64(out)
    assert_parity(got, ref, "large window T=512, every token")
    for t in range(T):
        assert_parity(got[t:t + 1], ref[t:t + 1], f"large window T=512, token {t}")


# ----------------------------------------------------------------- timeouts ---
def test_bounded_wait_runs_out_and_next_call_is_clean():
    """The kernels' wait limit shortened to 1 us: the layer's first waits (for the first
    weight stage, about 2 us after launch) run out, the call returns with MOE_ERR_TIMEOUT
    in the error word, and with the default limit back and the workspace's counter region
    cleared the next call matches the oracle.  The failure is made through the limit;
    nothing faults or hangs."""
    T, k, E, Hs, Is = 4, 8, 64, 4096, 2048
    L = make_layer(T, k, E, Hs, Is, seed=6400)
    bank = to_dev_bank(L)
    x, idx, w = to_dev_inputs(L)
    ws = qeg.moe_workspace(T, k, E, Hs, Is)
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    qeg.moe_set_wait_limit_ns(1000)
    try:
        qeg.moe_switchglu_forward_ws(x, idx, w, bank, ws)
        assert qeg.moe_read_device_status() == qeg.MOE_ERR_TIMEOUT
    finally:
        qeg.moe_set_wait_limit_ns(0)
    assert qeg.moe_read_device_status() == qeg.MOE_OK  # the read cleared the word
    ws[:4 * 1539].zero_()  # the caller clears its workspace after a timeout
    out = qeg.moe_switchglu_forward_ws(x, idx, w, bank, ws)
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    assert_parity(bf16_to_f64(out), oracle.switchglu(L.x, L.idx, L.w, L.bank, E),
                  "after a timeout")


# ------------------------------------------------------ router fused with the layer ---
@pytest.mark.parametrize("T,E,renorm", [(1, 288, True), (4, 288, True), (16, 288, False),
                                        (64, 288, True)])
def test_router_fused_into_the_layer(T, E, renorm):
    """Logits -> picks -> layer in one launch, against the router kernel then the layer (bit
    for bit: the same picks, weights and arithmetic) and against the oracle on sampled
    tokens; ties in the logits (equal values, the lower id first) included."""
    k, seed = 8, 4100 + T
    rng = np.random.default_rng(seed)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[:, 5] = lg[:, 6] = lg[:, 200] = 3.0  # equal logits among the top picks
    bank = dev_bank_drawn(E, H, I, seed)
    x_bits = synth.x_bf16(T, H, seed)
    x = bf16_tensor(x_bits)
    lgd = torch.from_numpy(lg).cuda()
    ws = qeg.moe_workspace(T, k, E, H, I)
    out, idx, w = qeg.moe_switchglu_forward_routed(x, lgd, k, bank, renormalize=renorm,
                                                   workspace=ws)
    idx2, w2 = qeg.moe_router_topk(lgd, k, renormalize=renorm)
    out2 = qeg.moe_switchglu_forward(x, idx2, w2, bank)
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    ridx, rw = oracle.router_topk(lg, k, renormalize=renorm)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=2e-5, atol=0)
    tokens = sample_tokens(T, 4, seed)
    used = sorted(set(int(e) for e in ridx[tokens].ravel()))
    hb = draw_bank(E, H, I, seed, used)
    ref = oracle.switchglu(x_bits, ridx, rw.astype(np.float32), hb, E, tokens=tokens)
    assert_parity(bf16_to_f64(out)[tokens], ref[tokens], f"router fused, T={T}")


def test_router_fused_grouped_path():
    """A window that takes the grouped path: the router kernel runs first, then the five
    grouped launches; the picks and output equal the two-call sequence's bit for bit."""
    T, k, E, Hs, Is = 160, 8, 64, 512, 256
    assert qeg.moe_select_path(T, k, E, Hs, Is) == 2
    L = make_layer(T, k, E, Hs, Is, 4300)
    bank = to_dev_bank(L)
    x, _, _ = to_dev_inputs(L)
    lg = torch.from_numpy(np.random.default_rng(4301).standard_normal((T, E))
                          .astype(np.float32)).cuda()
    out, idx, w = qeg.moe_switchglu_forward_routed(x, lg, k, bank)
    idx2, w2 = qeg.moe_router_topk(lg, k)
    out2 = qeg.moe_switchglu_forward(x, idx2, w2, bank)
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_one_token_with_repeated_experts_full_width():
    """A one-token window whose row names some experts more than once (segments of two
    and three pairs) at hidden 4096 / inter 2048: the one-token instance runs such a
    segment one pair per pass."""
    E, seed = 288, 4400
    idx = np.array([[5, 5, 17, 17, 17, 40, 41, 287]], np.int32)
    w = np.array([[0.2, 0.1, 0.15, 0.05, 0.1, 0.2, 0.1, 0.1]], np.float32)
    bank = dev_bank_drawn(E, H, I, seed)
    x_bits = synth.x_bf16(1, H, seed)
    check_sampled(x_bits, idx, w, bank, E, seed, [0], "one token, repeated experts")

