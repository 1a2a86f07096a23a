"""Oracle for the union-of-experts quantized SwitchGLU layer (fp64, CPU).

TEST INFRASTRUCTURE ONLY: a plain, slow, obviously correct restatement of what
the layer computes, used by tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  The product path
never imports it, and it shares no code with the CUDA library.

The arithmetic lives in ``oracle.cpp`` (see its header for the passages of the
pages it follows and the readings taken where they are silent).  This module
only builds it with g++ and marshals numpy arrays.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force, invariants and library special cases).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_SO = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(src: str = _SRC, so: str = _SO) -> str:
    """Compile oracle.cpp into a shared library (no-op when up to date)."""
    if not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-ffp-contract=off", "-o", so, src])
    return so


def load(so: Optional[str] = None):
    """Load the oracle library (building it first); `so` selects another build."""
    global _lib
    if so is None and _lib is not None:
        return _lib
    path = so or build()
    lib = ctypes.CDLL(path)
    vp, ci = ctypes.c_void_p, ctypes.c_int
    lib.oracle_route_union.restype = ci
    lib.oracle_route_union.argtypes = [vp, ci, ci, ci, vp, vp, vp, vp]
    lib.oracle_switchglu.restype = None
    lib.oracle_switchglu.argtypes = [vp] * 12 + [ci] * 5 + [vp, ci, ci, vp, vp, vp]
    lib.oracle_switchglu_union.restype = None
    lib.oracle_switchglu_union.argtypes = [vp] * 12 + [ci] * 5 + [vp, vp]
    lib.oracle_round_bf16.restype = ctypes.c_double
    lib.oracle_round_bf16.argtypes = [ctypes.c_double]
    lib.oracle_router_topk.restype = None
    lib.oracle_router_topk.argtypes = [vp, ci, ci, ci, ci, vp, vp]
    lib.oracle_switchglu_mxfp4.restype = None
    lib.oracle_switchglu_mxfp4.argtypes = [vp] * 9 + [ci] * 5 + [vp, ci, ci, vp, vp, vp]
    lib.oracle_mxfp4_value.restype = ctypes.c_double
    lib.oracle_mxfp4_value.argtypes = [ci, ci]
    if so is None:
        _lib = lib
    return lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def route_union(idx: np.ndarray, E: int, lib=None):
    """(unique[u], offsets[u+1], pair_list[P], u, invalid) for topk ids idx [T, k]."""
    lib = lib or load()
    idx, pidx = _c(idx, np.int32)
    T, k = idx.shape
    P = T * k
    m = max(1, min(E, P))
    uniq = np.zeros(m, np.int32)
    offs = np.zeros(m + 1, np.int32)
    plist = np.zeros(max(1, P), np.int32)
    u = np.zeros(1, np.int32)
    bad = lib.oracle_route_union(pidx, T, k, E, uniq.ctypes.data, offs.ctypes.data,
                                 plist.ctypes.data, u.ctypes.data)
    n = int(u[0])
    return uniq[:n].copy(), offs[:n + 1].copy(), plist[:P].copy(), n, int(bad)


def _bank_ptrs(bank):
    arrs = []
    for (q, s, b) in (bank["gate"], bank["up"], bank["down"]):
        arrs += [np.ascontiguousarray(q, np.uint32), np.ascontiguousarray(s, np.uint16),
                 np.ascontiguousarray(b, np.uint16)]
    return arrs


def switchglu(x: np.ndarray, idx: np.ndarray, w: np.ndarray, bank: dict, E: int,
              tokens: Optional[Sequence[int]] = None, n_threads: Optional[int] = None,
              want_h: bool = False, want_y: bool = False, lib=None):
    """Per-pair fp64 forward.  x [T,H] bf16 bits, idx [T,k] int32, w [T,k] f32,
    bank = {"gate": (q,s,b), "up": ..., "down": ...}.  Returns out [T,H] f64 (rows
    of unselected tokens are NaN), plus h [T*k, I] and/or y [T*k, H] if asked."""
    lib = lib or load()
    x, px = _c(x, np.uint16)
    idx, pidx = _c(idx, np.int32)
    w, pw = _c(w, np.float32)
    T, H = x.shape
    k = idx.shape[1]
    I = bank["gate"][0].shape[1]
    arrs = _bank_ptrs(bank)
    out = np.full((T, H), np.nan)
    h = np.zeros((T * k, I)) if want_h else None
    y = np.zeros((T * k, H)) if want_y else None
    tok = None if tokens is None else np.ascontiguousarray(tokens, np.int32)
    lib.oracle_switchglu(px, pidx, pw, *[a.ctypes.data for a in arrs], T, k, E, H, I,
                         None if tok is None else tok.ctypes.data,
                         0 if tok is None else int(tok.size),
                         n_threads or (os.cpu_count() or 1), out.ctypes.data,
                         None if h is None else h.ctypes.data, None if y is None else y.ctypes.data)
    res = [out]
    if want_h:
        res.append(h)
    if want_y:
        res.append(y)
    return res[0] if len(res) == 1 else tuple(res)


def switchglu_union(x, idx, w, bank, E, want_h=False, lib=None):
    """Deduplicated fp64 forward (single-threaded; small sizes only)."""
    lib = lib or load()
    x, px = _c(x, np.uint16)
    idx, pidx = _c(idx, np.int32)
    w, pw = _c(w, np.float32)
    T, H = x.shape
    k = idx.shape[1]
    I = bank["gate"][0].shape[1]
    arrs = _bank_ptrs(bank)
    out = np.zeros((T, H))
    h = np.zeros((T * k, I))
    lib.oracle_switchglu_union(px, pidx, pw, *[a.ctypes.data for a in arrs], T, k, E, H, I,
                               out.ctypes.data, h.ctypes.data)
    return (out, h) if want_h else out


def round_bf16(v: float, lib=None) -> float:
    return (lib or load()).oracle_round_bf16(float(v))


def router_topk(logits: np.ndarray, k: int, renormalize: bool = True, lib=None):
    """(idx [T, k] int32, w [T, k] fp64): top-k of softmax over each row of the fp32
    logits [T, E], descending, lower expert id first among equal logits; weights
    renormalised over the k unless renormalize is False."""
    lib = lib or load()
    logits, pl = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    lib.oracle_router_topk(pl, T, E, k, 1 if renormalize else 0, idx.ctypes.data, w.ctypes.data)
    return idx, w


def mxfp4_value(code: int, scale: int, lib=None) -> float:
    """The oracle's value of one mxfp4 weight: e2m1 code (0..15) times 2^(scale - 127)."""
    return (lib or load()).oracle_mxfp4_value(int(code), int(scale))


def switchglu_mxfp4(x, idx, w, bank: dict, E: int, tokens=None, want_h=False, lib=None):
    """The layer on mxfp4 banks: bank = {"gate": (q, e8), "up": (q, e8), "down": (q, e8)}
    with q uint32 [E, rows, cols/8] (e2m1 codes) and e8 uint8 [E, rows, cols/32]
    (e8m0 scales).  Same outputs as switchglu: out [T, H] fp64 (and h [T*k, I])."""
    lib = lib or load()
    x, px = _c(x, np.uint16)
    idx, pidx = _c(idx, np.int32)
    w, pw = _c(w, np.float32)
    T, H = x.shape
    k = idx.shape[1]
    I = bank["gate"][0].shape[1]
    arrs = []
    for name in ("gate", "up", "down"):
        q, e8 = bank[name]
        arrs.append(_c(q, np.uint32))
        arrs.append(_c(e8, np.uint8))
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    out = np.zeros((T, H), np.float64)
    h = np.zeros((T * k, I), np.float64) if want_h else None
    lib.oracle_switchglu_mxfp4(px, pidx, pw, *[a[1] for a in arrs], T, k, E, H, I,
                               None if tok is None else tok.ctypes.data,
                               0 if tok is None else len(tok), os.cpu_count() or 1,
                               out.ctypes.data, None if h is None else h.ctypes.data, None)
    return (out, h) if want_h else out

