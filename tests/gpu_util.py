"""Helpers for the GPU tests: upload seeded layers and compare against the oracle."""
from __future__ import annotations

import numpy as np
import torch

import quantized_expert_gather_b200 as qeg

# Parity bar for the bf16 layer output: rel-L2 = |out - ref| / |ref| over the whole
# output, and max-abs measured on the unit-RMS scale of the reference (max |out - ref|
# / rms(ref)), since the raw output of N(0,1) weights and inputs has an RMS near 1e5,
# where one bf16 step is already far above an absolute 3e-2.
REL_L2_TOL = 5e-3
MAX_ABS_TOL = 3e-2


def to_dev_bank(L, device="cuda") -> qeg.QuantBank:
    """Upload a host bank (tests.layers.Layer.bank) as a QuantBank of E experts."""
    t = {}
    for name, key in (("gate", "wg"), ("up", "wu"), ("down", "wd")):
        q, s, b = L.bank[name]
        t[key + "_q"] = torch.from_numpy(q.view(np.int32)).to(device)
        t[key + "_s"] = torch.from_numpy(s.view(np.int16)).to(device).view(torch.bfloat16)
        t[key + "_b"] = torch.from_numpy(b.view(np.int16)).to(device).view(torch.bfloat16)
    return qeg.QuantBank(**t)


def to_dev_inputs(L, device="cuda"):
    x = torch.from_numpy(L.x.view(np.int16)).to(device).view(torch.bfloat16)
    idx = torch.from_numpy(L.idx).to(device)
    w = torch.from_numpy(L.w).to(device)
    return x, idx, w


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def parity_errors(out: np.ndarray, ref: np.ndarray):
    """(relative L2 error, max-abs error over rms(ref), raw max-abs error)."""
    diff = out - ref
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.abs(diff).max()) if diff.size else 0.0
    return rel, (mx / rms if rms > 0 else mx), mx


def assert_parity(out: np.ndarray, ref: np.ndarray, what: str = ""):
    if not np.any(ref):
        assert not np.any(out), f"{what}: expected an all-zero output"
        return
    rel, mxn, mx = parity_errors(out, ref)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    assert rel <= REL_L2_TOL and mxn <= MAX_ABS_TOL, (
        f"{what}: rel-L2 {rel:.3e} (tol {REL_L2_TOL}), max-abs/rms {mxn:.3e} (tol {MAX_ABS_TOL}),"
        f" raw max-abs {mx:.3e}")


def dev_bank_drawn(E: int, H: int, I: int, seed: int, device="cuda") -> qeg.QuantBank:
    """A bank of E experts drawn on the device by the generator's CUDA twin, bit-identical
    to tests.layers.draw_bank(E, H, I, seed) (checked by a GPU test), so that the oracle
    can draw on the host only the experts a check needs."""
    import synth

    def mat(rows, cols, mid):
        q = torch.empty((E, rows, cols // 8), dtype=torch.int32, device=device)
        s = torch.empty((E, rows, cols // 64), dtype=torch.int16, device=device)
        b = torch.empty_like(s)
        synth.fill_bank_device(q, s, b, rows, cols, seed, mid)
        return q, s.view(torch.bfloat16), b.view(torch.bfloat16)

    bank = qeg.QuantBank(*mat(I, H, synth.MATRIX_GATE), *mat(I, H, synth.MATRIX_UP),
                         *mat(H, I, synth.MATRIX_DOWN))
    torch.cuda.synchronize()
    return bank


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """Device bf16 tensor from raw bf16 bit patterns (uint16)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device) \
        .view(torch.bfloat16)
