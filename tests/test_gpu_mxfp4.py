"""Parity of the mxfp4 layer (e2m1 codes, one e8m0 scale per 32 columns) against the
oracle's mxfp4 SwitchGLU.  The bank format is GLM-5.2's routed "mxfp4 gs32" ("Small-L fused
expert gather for fine-grained MoE decode", mlx discussion 3801, the post that isolates one
layer's routed bank: 256 experts of 3 x 6144 x 2048, ~20 MB per expert)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_gather_b200 as qeg
import synth
from tests.gpu_util import assert_parity, bf16_tensor, bf16_to_f64

pytestmark = pytest.mark.gpu


def host_bank(E, H, I, seed, experts=None):
    return {"gate": synth.fill_bank_mxfp4_host(E, I, H, seed, synth.MATRIX_GATE, experts),
            "up": synth.fill_bank_mxfp4_host(E, I, H, seed, synth.MATRIX_UP, experts),
            "down": synth.fill_bank_mxfp4_host(E, H, I, seed, synth.MATRIX_DOWN, experts)}


def dev_bank(E, H, I, seed):
    def mat(rows, cols, mid):
        q = torch.empty((E, rows, cols // 8), dtype=torch.int32, device="cuda")
        e8 = torch.empty((E, rows, cols // 32), dtype=torch.uint8, device="cuda")
        synth.fill_bank_mxfp4_device(q, e8, rows, cols, seed, mid)
        return q, e8
    b = qeg.MxBank(*mat(I, H, synth.MATRIX_GATE), *mat(I, H, synth.MATRIX_UP),
                   *mat(H, I, synth.MATRIX_DOWN))
    torch.cuda.synchronize()
    return b


def upload(hb):
    t = []
    for name in ("gate", "up", "down"):
        q, e8 = hb[name]
        t += [torch.from_numpy(q.view(np.int32)).cuda(), torch.from_numpy(e8).cuda()]
    return qeg.MxBank(*t)


def run(x_bits, idx, w, bank):
    out = qeg.moe_switchglu_forward_mxfp4(bf16_tensor(x_bits), torch.from_numpy(idx).cuda(),
                                          torch.from_numpy(w).cuda(), bank)
    torch.cuda.synchronize()
    return out


def test_device_generator_matches_host_mxfp4():
    E, rows, cols, seed = 4, 48, 512, 91
    q = torch.zeros((E, rows, cols // 8), dtype=torch.int32, device="cuda")
    e8 = torch.zeros((E, rows, cols // 32), dtype=torch.uint8, device="cuda")
    synth.fill_bank_mxfp4_device(q, e8, rows, cols, seed, synth.MATRIX_GATE)
    torch.cuda.synchronize()
    qh, eh = synth.fill_bank_mxfp4_host(E, rows, cols, seed, synth.MATRIX_GATE)
    assert np.array_equal(q.cpu().numpy().view(np.uint32), qh)
    assert np.array_equal(e8.cpu().numpy(), eh)


@pytest.mark.parametrize("cfg", [
    # T, k, E, H, I
    (2, 2, 16, 256, 128),
    (7, 6, 40, 512, 384),
    (5, 3, 8, 1024, 576),
    (16, 8, 64, 768, 256),
])
def test_mxfp4_small_shapes(cfg):
    T, k, E, H, I = cfg
    seed = 7000 + sum(cfg)
    idx, w = synth.route_uniform(T, E, k, seed)
    hb = host_bank(E, H, I, seed)
    x = synth.x_bf16(T, H, seed)
    out = run(x, idx, w, upload(hb))
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    assert_parity(bf16_to_f64(out), oracle.switchglu_mxfp4(x, idx, w, hb, E),
                  f"mxfp4 T={T} k={k} E={E} H={H} I={I}")


@pytest.mark.parametrize("T", [1, 2, 4, 16])
def test_mxfp4_glm52_bank(T):
    """E=256, top-8, hidden 6144, intermediate 2048 (GLM-5.2's routed bank), adjacent-overlap
    routing at p = 0.34; every token against the oracle."""
    E, H, I, seed = 256, 6144, 2048, 7100 + T
    bank = dev_bank(E, H, I, seed)
    idx, w = synth.route_markov(T, E, 8, 0.34, seed)
    x = synth.x_bf16(T, H, seed)
    out = run(x, idx, w, bank)
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    used = sorted(set(int(e) for e in idx.ravel()))
    ref = oracle.switchglu_mxfp4(x, idx, w, host_bank(E, H, I, seed, used), E)
    assert_parity(bf16_to_f64(out), ref, f"mxfp4 GLM-5.2 bank T={T}")


@pytest.mark.parametrize("cfg", [
    # T, k, E, H, I: more than 1024 pairs, so the grouped tensor-core path
    (160, 8, 64, 512, 256),
    (200, 6, 32, 768, 384),
    (600, 2, 3, 256, 128),   # about 400 pairs per expert: several chunks of 96
])
def test_mxfp4_grouped_small_shapes(cfg):
    T, k, E, H, I = cfg
    assert qeg.moe_select_path_mxfp4(T, k, E, H, I) == 2
    seed = 7200 + sum(cfg)
    idx, w = synth.route_uniform(T, E, k, seed)
    hb = host_bank(E, H, I, seed)
    x = synth.x_bf16(T, H, seed)
    out = run(x, idx, w, upload(hb))
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    assert_parity(bf16_to_f64(out), oracle.switchglu_mxfp4(x, idx, w, hb, E),
                  f"mxfp4 grouped T={T} k={k} E={E} H={H} I={I}")


def test_mxfp4_glm52_bank_large_window():
    """GLM-5.2's routed bank (E=256, 6144 x 2048) at T=512 with uniform top-8 routing: the
    grouped path; sampled tokens against the oracle."""
    E, H, I, T, seed = 256, 6144, 2048, 512, 7300
    assert qeg.moe_select_path_mxfp4(T, 8, E, H, I) == 2
    bank = dev_bank(E, H, I, seed)
    idx, w = synth.route_uniform(T, E, 8, seed)
    x = synth.x_bf16(T, H, seed)
    out = run(x, idx, w, bank)
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    tokens = sorted(np.random.default_rng(seed).choice(T, 8, replace=False).tolist())
    used = sorted(set(int(e) for e in idx[tokens].ravel()))
    ref = oracle.switchglu_mxfp4(x[tokens], idx[tokens], w[tokens],
                                 host_bank(E, H, I, seed, used), E)
    assert_parity(bf16_to_f64(out)[tokens], ref, "mxfp4 GLM-5.2 bank T=512 (sampled tokens)")
