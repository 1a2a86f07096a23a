"""Seeded synthetic inputs for the union-of-experts quantized SwitchGLU layer.

Inputs only: this package holds none of the layer's arithmetic.  Both the
oracle and the CUDA path consume what it draws.

* Expert banks: ``fill_bank_host`` (C, threaded) and ``fill_bank_device``
  (CUDA) implement one counter-based generator and one quantiser and produce the
  same bits (see ``synth_host.c`` for the definition).  ``fill_bank_mxfp4_host`` /
  ``fill_bank_mxfp4_device`` encode the same draws as mxfp4 (e2m1 codes, one e8m0
  scale per 32 columns).  The 4-bit affine
  group-64 format with bf16 scale and bias is the one of the ``moe_bench.py``
  script in "gather_qmm at M=1 streams 4-bit expert weights at ~half the
  bandwidth of M=4" (mlx issue 4509).
* Activations: N(0,1) fp32 draws rounded to bf16 (round to nearest even).
* Routing models (numpy ``default_rng``):

  - ``route_softmax_topk``: top-k of softmax(N(0,1) logits), weights renormalised
    over the chosen k (the tiny parity layer).
  - ``route_uniform``: each token's k experts drawn uniformly without
    replacement, like ``random.sample(range(E), TOPK)`` in the moe_bench.py
    script; weights softmax of N(0,1) logits over the chosen k.
  - ``route_verify_pair`` / ``route_markov``: token t+1 keeps each of token t's
    experts with probability p and draws the rest uniformly without
    replacement from the experts token t did not use, so the adjacent-token
    overlap is p on average (the overlap statistic of "Small-L fused expert
    gather for fine-grained MoE decode", mlx discussion 3801: 34.1 % mean,
    3 % at random, up to 52 % in deep layers).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "libsynth_host.so")
_DEV_SO = os.path.join(_HERE, "libsynth_dev.so")

MATRIX_GATE, MATRIX_UP, MATRIX_DOWN = 0, 1, 2


def build(device: bool = True) -> None:
    """Compile the host generator (gcc) and, if requested, the device twin (nvcc)."""
    src = os.path.join(_HERE, "synth_host.c")
    if not os.path.exists(_HOST_SO) or os.path.getmtime(_HOST_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                               "-pthread", "-o", _HOST_SO, src, "-lm"])
    if device:
        dsrc = os.path.join(_HERE, "synth_dev.cu")
        if not os.path.exists(_DEV_SO) or os.path.getmtime(_DEV_SO) < os.path.getmtime(dsrc):
            subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                                   "-fmad=false", "-Xcompiler", "-fPIC", "-shared", "-o", _DEV_SO,
                                   dsrc])


_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        build(device=False)
        lib = ctypes.CDLL(_HOST_SO)
        lib.synth_fill_bank.restype = ctypes.c_int
        lib.synth_fill_bank.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p,
                                        ctypes.c_int, ctypes.c_int]
        lib.synth_fill_bank_mxfp4.restype = ctypes.c_int
        lib.synth_fill_bank_mxfp4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                              ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int,
                                              ctypes.c_int]
        lib.synth_draw_row.restype = ctypes.c_int
        lib.synth_draw_row.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int,
                                       ctypes.c_int]
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        build(device=True)
        lib = ctypes.CDLL(_DEV_SO)
        lib.synth_dev_fill_bank.restype = ctypes.c_int
        lib.synth_dev_fill_bank.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                            ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int,
                                            ctypes.c_void_p]
        lib.synth_dev_fill_bank_mxfp4.restype = ctypes.c_int
        lib.synth_dev_fill_bank_mxfp4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64,
                                                  ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
        _dev = lib
    return _dev


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else
               (os.cpu_count() or 1))


def alloc_bank(E: int, rows: int, cols: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Zeroed host bank arrays q [E,rows,cols/8] u32, s/b [E,rows,cols/64] bf16 bits."""
    return (np.zeros((E, rows, cols // 8), np.uint32), np.zeros((E, rows, cols // 64), np.uint16),
            np.zeros((E, rows, cols // 64), np.uint16))


def fill_bank_host(E: int, rows: int, cols: int, seed: int, matrix_id: int,
                   experts: Optional[Sequence[int]] = None, n_threads: Optional[int] = None,
                   out=None):
    """Draw experts `experts` (default: all) of one matrix of a bank on the host.

    Returns (q, s, b) numpy arrays; experts not listed stay zero (or untouched if
    `out` is given).
    """
    if cols % 64:
        raise ValueError("cols must be a multiple of 64")
    q, s, b = out if out is not None else alloc_bank(E, rows, cols)
    ex = np.arange(E, dtype=np.int32) if experts is None else np.asarray(
        sorted(set(int(e) for e in experts)), dtype=np.int32)
    if ex.size:
        rc = _host_lib().synth_fill_bank(q.ctypes.data, s.ctypes.data, b.ctypes.data, E, rows,
                                         cols, seed, matrix_id, ex.ctypes.data, int(ex.size),
                                         n_threads or default_threads())
        if rc != 0:
            raise ValueError("synth_fill_bank rejected its arguments")
    return q, s, b


def alloc_bank_mxfp4(E: int, rows: int, cols: int) -> Tuple[np.ndarray, np.ndarray]:
    """Zeroed host mxfp4 bank arrays q [E,rows,cols/8] u32 (e2m1 codes), e8 [E,rows,cols/32]
    u8 (e8m0 scales)."""
    return np.zeros((E, rows, cols // 8), np.uint32), np.zeros((E, rows, cols // 32), np.uint8)


def fill_bank_mxfp4_host(E: int, rows: int, cols: int, seed: int, matrix_id: int,
                         experts: Optional[Sequence[int]] = None,
                         n_threads: Optional[int] = None, out=None):
    """Draw experts `experts` (default: all) of one matrix of an mxfp4 bank on the host
    (the same normal draws as fill_bank_host, encoded as e2m1 codes with one e8m0 scale
    per 32 columns; see synth_host.c).  Returns (q, e8)."""
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    q, e8 = out if out is not None else alloc_bank_mxfp4(E, rows, cols)
    ex = np.arange(E, dtype=np.int32) if experts is None else np.asarray(
        sorted(set(int(e) for e in experts)), dtype=np.int32)
    if ex.size:
        rc = _host_lib().synth_fill_bank_mxfp4(q.ctypes.data, e8.ctypes.data, E, rows, cols, seed,
                                               matrix_id, ex.ctypes.data, int(ex.size),
                                               n_threads or default_threads())
        if rc != 0:
            raise ValueError("synth_fill_bank_mxfp4 rejected its arguments")
    return q, e8


def fill_bank_mxfp4_device(q, e8, rows: int, cols: int, seed: int, matrix_id: int,
                           experts=None, n_experts: Optional[int] = None,
                           stream: int = 0) -> None:
    """Draw an mxfp4 bank into device tensors q (int32 [E,rows,cols/8]) and e8 (uint8
    [E,rows,cols/32]), bit-identical to fill_bank_mxfp4_host."""
    n = int(experts.numel()) if experts is not None else int(n_experts or q.shape[0])
    rc = _dev_lib().synth_dev_fill_bank_mxfp4(q.data_ptr(), e8.data_ptr(), rows, cols, seed,
                                              matrix_id,
                                              experts.data_ptr() if experts is not None else None,
                                              n, stream)
    if rc != 0:
        raise RuntimeError(f"synth_dev_fill_bank_mxfp4 failed with code {rc}")


def draw_row(E: int, rows: int, cols: int, seed: int, matrix_id: int, expert: int,
             row: int) -> np.ndarray:
    """The fp32 N(0,1) draws of one row before quantisation."""
    out = np.empty(cols, np.float32)
    if _host_lib().synth_draw_row(out.ctypes.data, E, rows, cols, seed, matrix_id, expert,
                                  row) != 0:
        raise ValueError("bad row")
    return out


def fill_bank_device(q, s, b, rows: int, cols: int, seed: int, matrix_id: int,
                     experts=None, n_experts: Optional[int] = None, stream: int = 0) -> None:
    """Draw a bank directly into device tensors (torch) q/s/b, bit-identical to the host.

    `experts` is an optional device int32 tensor of expert ids; without it experts
    0..n_experts-1 (default: q.shape[0]) are drawn.
    """
    n = int(experts.numel()) if experts is not None else int(n_experts or q.shape[0])
    rc = _dev_lib().synth_dev_fill_bank(q.data_ptr(), s.data_ptr(), b.data_ptr(), rows, cols,
                                        seed, matrix_id,
                                        experts.data_ptr() if experts is not None else None, n,
                                        stream)
    if rc != 0:
        raise RuntimeError(f"synth_dev_fill_bank failed with code {rc}")


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest even); returns the raw 16-bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    special = (u & 0x7F800000) == 0x7F800000
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[special] = (u[special] >> 16).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def x_bf16(T: int, H: int, seed: int) -> np.ndarray:
    """Activations [T, H]: N(0,1) fp32 draws rounded to bf16 (raw uint16 bits)."""
    rng = np.random.default_rng([seed, 0x5EED])
    return f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))


def _softmax(z: np.ndarray) -> np.ndarray:
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def route_softmax_topk(T: int, E: int, k: int, seed: int):
    """Top-k of softmax(N(0,1) logits) per token, weights renormalised over the k.

    Ties (measure zero) go to the lower expert index.
    """
    rng = np.random.default_rng([seed, 0xA11CE])
    logits = rng.standard_normal((T, E))
    p = _softmax(logits)
    idx = np.argsort(-p, axis=-1, kind="stable")[:, :k]
    w = np.take_along_axis(p, idx, axis=-1)
    w = w / w.sum(axis=-1, keepdims=True)
    return idx.astype(np.int32), w.astype(np.float32)


def _weights_over_chosen(rng, T: int, k: int) -> np.ndarray:
    return _softmax(rng.standard_normal((T, k))).astype(np.float32)


def route_uniform(T: int, E: int, k: int, seed: int):
    """Each token's k experts uniformly without replacement (sorted ascending within
    the token, as the moe_bench.py script does); weights softmax(N(0,1)) over the k."""
    rng = np.random.default_rng([seed, 0xB0B])
    idx = np.stack([np.sort(rng.choice(E, size=k, replace=False)) for _ in range(T)])
    return idx.astype(np.int32), _weights_over_chosen(rng, T, k)


def _next_token(rng, prev: np.ndarray, E: int, k: int, p: float) -> np.ndarray:
    keep = prev[rng.random(k) < p]
    pool = np.setdiff1d(np.arange(E), prev)
    fresh = rng.choice(pool, size=k - keep.size, replace=False)
    return np.sort(np.concatenate([keep, fresh]))


def route_markov(T: int, E: int, k: int, p: float, seed: int):
    """Adjacent-overlap chain: token 0 uniform; token t+1 keeps each of token t's
    experts with probability p and fills the other slots uniformly without
    replacement from the E-k experts token t did not use."""
    if not 0.0 <= p <= 1.0:
        raise ValueError("p must be in [0, 1]")
    rng = np.random.default_rng([seed, 0xC4A1])
    rows = [np.sort(rng.choice(E, size=k, replace=False))]
    for _ in range(1, T):
        rows.append(_next_token(rng, rows[-1], E, k, p))
    return np.stack(rows).astype(np.int32), _weights_over_chosen(rng, T, k)


def route_verify_pair(E: int, k: int, p: float, seed: int):
    """The speculative-verify pair: a two-token chain of `route_markov`."""
    return route_markov(2, E, k, p, seed)
