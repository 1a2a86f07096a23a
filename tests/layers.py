"""Seeded test layers: banks, activations and routing drawn with ``synth``.

Shared by the oracle pins and the GPU parity tests.  Holds no layer arithmetic.
"""
from __future__ import annotations

import os
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np

import synth


@dataclass
class Layer:
    T: int
    k: int
    E: int
    H: int
    I: int
    x: np.ndarray                     # [T, H] bf16 bits
    idx: np.ndarray                   # [T, k] int32
    w: np.ndarray                     # [T, k] float32
    bank: Dict[str, Tuple[np.ndarray, np.ndarray, np.ndarray]] = field(default_factory=dict)
    seed: int = 0


def draw_bank(E: int, H: int, I: int, seed: int, experts=None):
    """Bank of E experts; only `experts` are drawn (others stay zero)."""
    return {
        "gate": synth.fill_bank_host(E, I, H, seed, synth.MATRIX_GATE, experts),
        "up": synth.fill_bank_host(E, I, H, seed, synth.MATRIX_UP, experts),
        "down": synth.fill_bank_host(E, H, I, seed, synth.MATRIX_DOWN, experts),
    }


def make_layer(T: int, k: int, E: int, H: int, I: int, seed: int, routing: str = "uniform",
               p: float = 0.4, idx: Optional[np.ndarray] = None, w: Optional[np.ndarray] = None,
               draw_all: bool = False) -> Layer:
    if idx is None:
        if routing == "softmax":
            idx, w = synth.route_softmax_topk(T, E, k, seed)
        elif routing == "uniform":
            idx, w = synth.route_uniform(T, E, k, seed)
        elif routing == "markov":
            idx, w = synth.route_markov(T, E, k, p, seed)
        else:
            raise ValueError(routing)
    if w is None:
        w = np.full((T, k), 1.0 / k, np.float32)
    used = None if draw_all else sorted(set(int(e) for e in idx.ravel() if 0 <= e < E))
    bank = draw_bank(E, H, I, seed, used)
    return Layer(T, k, E, H, I, synth.x_bf16(T, H, seed), np.ascontiguousarray(idx, np.int32),
                 np.ascontiguousarray(w, np.float32), bank, seed)


def tiny_layer() -> Layer:
    """E=16, top-2, hidden 256, intermediate 128, T=2, softmax top-2 routing, seed 0."""
    return make_layer(2, 2, 16, 256, 128, 0, routing="softmax", draw_all=True)


def read_golden(name: str) -> Dict[str, list]:
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
    out = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            out[parts[0]] = [float(v) for v in parts[1:]]
    return out
