"""Python binding of libmoe_qeg (include/moe_qeg.h): union-of-experts 4-bit
quantized MoE SwitchGLU layer for B200 (sm_100a).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The functions take torch CUDA tensors, check dtypes and shapes, and
pass raw pointers plus the current CUDA stream to the C entry points of the
same name.  If the compiled library is missing or cannot be loaded this module
raises on import: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from ._build import SO, build as build_library, needs_build

__all__ = ["MoeError", "MOE_OK", "moe_status_str", "moe_workspace_size", "moe_workspace_layout",
           "moe_select_path", "moe_route_union", "moe_switchglu_forward",
           "moe_switchglu_forward_ws", "moe_switchglu_forward_static", "moe_read_device_status", "moe_last_error", "moe_workspace",
           "library_path", "QuantBank", "MxBank", "moe_switchglu_forward_mxfp4",
           "moe_switchglu_forward_mxfp4_ws", "moe_workspace_size_mxfp4", "moe_select_path_mxfp4"]

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_DEVICE_INDEX = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_WORKSPACE = 6


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        detail = f" [{moe_last_error()}]" if status == MOE_ERR_CUDA else ""
        super().__init__(f"{where}: {moe_status_str(status)} ({status}){detail}")
        self.status = status


def _load():
    if needs_build():
        build_library()
    lib = ctypes.CDLL(SO)
    vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.moe_status_str.restype = ctypes.c_char_p
    lib.moe_status_str.argtypes = [ci]
    lib.moe_last_error.restype = ctypes.c_char_p
    lib.moe_last_error.argtypes = []
    lib.moe_workspace_size.restype = sz
    lib.moe_workspace_size.argtypes = [ci] * 5
    lib.moe_workspace_layout.restype = ci
    lib.moe_workspace_layout.argtypes = [ci] * 5 + [vp]
    lib.moe_select_path.restype = ci
    lib.moe_select_path.argtypes = [ci] * 5
    lib.moe_route_union.restype = ci
    lib.moe_route_union.argtypes = [vp, ci, ci, ci, vp, vp, vp, vp, vp]
    lib.moe_router_topk.restype = ci
    lib.moe_router_topk.argtypes = [vp, ci, ci, ci, ci, vp, vp, vp]
    lib.moe_switchglu_forward.restype = ci
    lib.moe_switchglu_forward.argtypes = [vp] * 12 + [ci] * 5 + [vp, vp]
    lib.moe_switchglu_forward_ws.restype = ci
    lib.moe_switchglu_forward_ws.argtypes = [vp] * 12 + [ci] * 5 + [vp, vp, sz, vp]
    lib.moe_switchglu_forward_static.restype = ci
    lib.moe_switchglu_forward_static.argtypes = [vp] * 12 + [ci] * 5 + [vp, vp]
    # (x, logits, renormalize, 9 bank pointers, T, k, E, hidden, inter, out, topk_idx,
    # topk_w, [workspace, bytes,] stream)
    lib.moe_switchglu_forward_routed.restype = ci
    lib.moe_switchglu_forward_routed.argtypes = [vp, vp, ci] + [vp] * 9 + [ci] * 5 + [vp] * 4
    lib.moe_switchglu_forward_routed_ws.restype = ci
    lib.moe_switchglu_forward_routed_ws.argtypes = ([vp, vp, ci] + [vp] * 9 + [ci] * 5 +
                                                    [vp] * 4 + [sz, vp])
    lib.moe_workspace_size_mxfp4.restype = sz
    lib.moe_workspace_size_mxfp4.argtypes = [ci] * 5
    lib.moe_select_path_mxfp4.restype = ci
    lib.moe_select_path_mxfp4.argtypes = [ci] * 5
    lib.moe_switchglu_forward_mxfp4.restype = ci
    lib.moe_switchglu_forward_mxfp4.argtypes = [vp] * 9 + [ci] * 5 + [vp, vp]
    lib.moe_switchglu_forward_mxfp4_ws.restype = ci
    lib.moe_switchglu_forward_mxfp4_ws.argtypes = [vp] * 9 + [ci] * 5 + [vp, vp, sz, vp]
    lib.moe_set_wait_limit_ns.restype = ci
    lib.moe_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.moe_read_device_status.restype = ci
    lib.moe_read_device_status.argtypes = [vp]
    return lib


_lib = _load()


def library_path() -> str:
    return SO


def moe_status_str(status: int) -> str:
    return _lib.moe_status_str(int(status)).decode()


def moe_last_error() -> str:
    return _lib.moe_last_error().decode()


def _check(status: int, where: str, check: bool) -> int:
    if check and status != MOE_OK:
        raise MoeError(status, where)
    return status


def _stream(stream, device=None) -> int:
    """The raw CUDA stream handle: `stream` itself, or the current stream of `device`."""
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _same_device(device, **tensors) -> None:
    """The library picks its per-device state (workspace, scratch, attributes) by the
    current device, so every tensor of a call must live on the device the call runs on."""
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, expected {device}")


def _ptr(t: torch.Tensor, dtypes, name: str) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)
_Q = (torch.int32, torch.uint32)
_I32 = (torch.int32,)
_F32 = (torch.float32,)
_U8 = (torch.uint8,)


def moe_workspace_size(T: int, k: int, E: int, hidden: int, inter: int) -> int:
    return int(_lib.moe_workspace_size(T, k, E, hidden, inter))


def moe_workspace_layout(T: int, k: int, E: int, hidden: int, inter: int) -> dict:
    out = (ctypes.c_size_t * 8)()
    _check(_lib.moe_workspace_layout(T, k, E, hidden, inter, ctypes.addressof(out)),
           "moe_workspace_layout", True)
    return dict(zip(("barrier", "num_unique", "unique", "offsets", "pair_list", "h", "y",
                     "total"), list(out)))


def moe_workspace(T: int, k: int, E: int, hidden: int, inter: int, device=None) -> torch.Tensor:
    """A zeroed uint8 device workspace of the size moe_switchglu_forward_ws needs."""
    return torch.zeros(moe_workspace_size(T, k, E, hidden, inter), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def moe_select_path(T: int, k: int, E: int, hidden: int, inter: int) -> int:
    return int(_lib.moe_select_path(T, k, E, hidden, inter))


def moe_route_union(topk_idx: torch.Tensor, E: int, unique=None, offsets=None, pair_list=None,
                    num_unique=None, stream=None, check: bool = True):
    """Route-union of topk_idx [T, k] (int32, CUDA).  Returns (unique, offsets, pair_list,
    num_unique) device tensors of sizes min(E,P), min(E,P)+1, P, 1."""
    T, k = topk_idx.shape
    P = T * k
    m = max(1, min(E, P))
    dev = topk_idx.device
    unique = unique if unique is not None else torch.zeros(m, dtype=torch.int32, device=dev)
    offsets = offsets if offsets is not None else torch.zeros(m + 1, dtype=torch.int32, device=dev)
    pair_list = pair_list if pair_list is not None else torch.zeros(P, dtype=torch.int32,
                                                                    device=dev)
    num_unique = num_unique if num_unique is not None else torch.zeros(1, dtype=torch.int32,
                                                                       device=dev)
    _same_device(dev, unique=unique, offsets=offsets, pair_list=pair_list, num_unique=num_unique)
    with torch.cuda.device(dev):
        st = _lib.moe_route_union(_ptr(topk_idx, _I32, "topk_idx"), T, k, E,
                                  _ptr(unique, _I32, "unique"), _ptr(offsets, _I32, "offsets"),
                                  _ptr(pair_list, _I32, "pair_list"),
                                  _ptr(num_unique, _I32, "num_unique"), _stream(stream, dev))
    _check(st, "moe_route_union", check)
    return unique, offsets, pair_list, num_unique


def moe_router_topk(logits: torch.Tensor, k: int, renormalize: bool = True, topk_idx=None,
                    topk_w=None, stream=None, check: bool = True):
    """Router step: top-k of softmax over each row of logits [T, E] (fp32, CUDA),
    descending, lower expert id first among equal logits; weights renormalised over
    the k unless renormalize is False.  Returns (topk_idx [T, k] int32, topk_w [T, k]
    fp32), the inputs of moe_switchglu_forward."""
    T, E = logits.shape
    dev = logits.device
    topk_idx = topk_idx if topk_idx is not None else torch.empty((T, k), dtype=torch.int32,
                                                                 device=dev)
    topk_w = topk_w if topk_w is not None else torch.empty((T, k), dtype=torch.float32,
                                                           device=dev)
    _same_device(dev, topk_idx=topk_idx, topk_w=topk_w)
    with torch.cuda.device(dev):
        st = _lib.moe_router_topk(_ptr(logits, _F32, "logits"), T, E, k, 1 if renormalize else 0,
                                  _ptr(topk_idx, _I32, "topk_idx"), _ptr(topk_w, _F32, "topk_w"),
                                  _stream(stream, dev))
    _check(st, "moe_router_topk", check)
    return topk_idx, topk_w


class QuantBank:
    """Device tensors of one layer's expert bank: gate/up q [E, inter, hidden/8],
    s/b [E, inter, hidden/64]; down q [E, hidden, inter/8], s/b [E, hidden, inter/64]."""

    def __init__(self, wg_q, wg_s, wg_b, wu_q, wu_s, wu_b, wd_q, wd_s, wd_b):
        self.wg_q, self.wg_s, self.wg_b = wg_q, wg_s, wg_b
        self.wu_q, self.wu_s, self.wu_b = wu_q, wu_s, wu_b
        self.wd_q, self.wd_s, self.wd_b = wd_q, wd_s, wd_b
        self.E, self.inter, hw = wg_q.shape
        self.hidden = hw * 8
        for name, t, shape in (("wg_s", wg_s, (self.E, self.inter, self.hidden // 64)),
                               ("wu_q", wu_q, wg_q.shape),
                               ("wd_q", wd_q, (self.E, self.hidden, self.inter // 8)),
                               ("wd_s", wd_s, (self.E, self.hidden, self.inter // 64))):
            if tuple(t.shape) != tuple(shape):
                raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")

    def ptrs(self):
        return [_ptr(self.wg_q, _Q, "wg_q"), _ptr(self.wg_s, _BF16, "wg_s"),
                _ptr(self.wg_b, _BF16, "wg_b"), _ptr(self.wu_q, _Q, "wu_q"),
                _ptr(self.wu_s, _BF16, "wu_s"), _ptr(self.wu_b, _BF16, "wu_b"),
                _ptr(self.wd_q, _Q, "wd_q"), _ptr(self.wd_s, _BF16, "wd_s"),
                _ptr(self.wd_b, _BF16, "wd_b")]


def _fwd_args(x, topk_idx, topk_w, bank: QuantBank, out):
    T, hidden = x.shape
    k = topk_idx.shape[1]
    if hidden != bank.hidden or tuple(topk_idx.shape) != (T, k) or tuple(topk_w.shape) != (T, k):
        raise ValueError("x / topk_idx / topk_w shapes do not match the bank")
    if out is None:
        out = torch.empty((T, hidden), dtype=torch.bfloat16, device=x.device)
    if tuple(out.shape) != (T, hidden):
        raise ValueError("out has the wrong shape")
    _same_device(x.device, topk_idx=topk_idx, topk_w=topk_w, out=out, wg_q=bank.wg_q,
                 wg_s=bank.wg_s, wg_b=bank.wg_b, wu_q=bank.wu_q, wu_s=bank.wu_s, wu_b=bank.wu_b,
                 wd_q=bank.wd_q, wd_s=bank.wd_s, wd_b=bank.wd_b)
    args = [_ptr(x, _BF16, "x"), _ptr(topk_idx, _I32, "topk_idx"), _ptr(topk_w, _F32, "topk_w"),
            *bank.ptrs()]
    return args, (T, k, bank.E, hidden, bank.inter), out


def moe_switchglu_forward(x, topk_idx, topk_w, bank: QuantBank, out=None, stream=None,
                          check: bool = True):
    """out [T, hidden] bf16 = union-of-experts SwitchGLU of x [T, hidden] bf16."""
    args, dims, out = _fwd_args(x, topk_idx, topk_w, bank, out)
    with torch.cuda.device(x.device):
        st = _lib.moe_switchglu_forward(*args, *dims, _ptr(out, _BF16, "out"),
                                        _stream(stream, x.device))
    _check(st, "moe_switchglu_forward", check)
    return out


def moe_switchglu_forward_ws(x, topk_idx, topk_w, bank: QuantBank, workspace: torch.Tensor,
                             out=None, stream=None, check: bool = True):
    """As moe_switchglu_forward, with a caller-owned uint8 device workspace tensor (see
    moe_workspace).  Its counter region (the first 4 * 1539 bytes) must be zero before the
    first call; the kernel leaves it zero again, except after a call that ended in
    MOE_ERR_TIMEOUT, when the caller must clear it before the next call."""
    args, dims, out = _fwd_args(x, topk_idx, topk_w, bank, out)
    _same_device(x.device, workspace=workspace)
    with torch.cuda.device(x.device):
        st = _lib.moe_switchglu_forward_ws(*args, *dims, _ptr(out, _BF16, "out"),
                                           _ptr(workspace, (torch.uint8,), "workspace"),
                                           workspace.numel(), _stream(stream, x.device))
    _check(st, "moe_switchglu_forward_ws", check)
    return out


def moe_switchglu_forward_static(x, topk_idx, topk_w, bank: QuantBank, out=None, stream=None,
                                 check: bool = True):
    """As moe_switchglu_forward, with the library's fixed per-device scratch (no allocation
    inside the call; shapes needing more than MOE_STATIC_SCRATCH_BYTES are rejected with
    MOE_ERR_WORKSPACE; overlapping calls on one device race)."""
    args, dims, out = _fwd_args(x, topk_idx, topk_w, bank, out)
    with torch.cuda.device(x.device):
        st = _lib.moe_switchglu_forward_static(*args, *dims, _ptr(out, _BF16, "out"),
                                               _stream(stream, x.device))
    if check and st == MOE_ERR_WORKSPACE:
        raise MoeError(st, f"moe_switchglu_forward_static [{moe_last_error()}]")
    _check(st, "moe_switchglu_forward_static", check)
    return out


def _routed_args(x, logits, k, bank: QuantBank, out, topk_idx, topk_w):
    T, hidden = x.shape
    if hidden != bank.hidden or logits.dim() != 2 or logits.shape[0] != T \
            or logits.shape[1] != bank.E:
        raise ValueError("x / logits shapes do not match the bank")
    dev = x.device
    out = out if out is not None else torch.empty((T, hidden), dtype=torch.bfloat16, device=dev)
    topk_idx = topk_idx if topk_idx is not None else torch.empty((T, k), dtype=torch.int32,
                                                                 device=dev)
    topk_w = topk_w if topk_w is not None else torch.empty((T, k), dtype=torch.float32,
                                                           device=dev)
    if tuple(out.shape) != (T, hidden) or tuple(topk_idx.shape) != (T, k) \
            or tuple(topk_w.shape) != (T, k):
        raise ValueError("out / topk_idx / topk_w have the wrong shape")
    _same_device(dev, logits=logits, out=out, topk_idx=topk_idx, topk_w=topk_w, wg_q=bank.wg_q,
                 wd_q=bank.wd_q)
    return out, topk_idx, topk_w


def moe_switchglu_forward_routed(x, logits, k: int, bank: QuantBank, renormalize: bool = True,
                                 workspace=None, out=None, topk_idx=None, topk_w=None,
                                 stream=None, check: bool = True):
    """The router step and the layer in one call: picks of top-k of softmax over each row of
    logits [T, E] (fp32, CUDA) as moe_router_topk makes them, then the layer on those picks.
    Returns (out [T, hidden] bf16, topk_idx [T, k] int32, topk_w [T, k] fp32).  With
    `workspace` (see moe_workspace) the call uses it, else the library-owned one."""
    out, topk_idx, topk_w = _routed_args(x, logits, k, bank, out, topk_idx, topk_w)
    T, hidden = x.shape
    dims = (T, k, bank.E, hidden, bank.inter)
    head = [_ptr(x, _BF16, "x"), _ptr(logits, _F32, "logits"), 1 if renormalize else 0,
            *bank.ptrs()]
    tail = [_ptr(out, _BF16, "out"), _ptr(topk_idx, _I32, "topk_idx"),
            _ptr(topk_w, _F32, "topk_w")]
    with torch.cuda.device(x.device):
        if workspace is None:
            st = _lib.moe_switchglu_forward_routed(*head, *dims, *tail, _stream(stream, x.device))
            name = "moe_switchglu_forward_routed"
        else:
            _same_device(x.device, workspace=workspace)
            st = _lib.moe_switchglu_forward_routed_ws(
                *head, *dims, *tail, _ptr(workspace, (torch.uint8,), "workspace"),
                workspace.numel(), _stream(stream, x.device))
            name = "moe_switchglu_forward_routed_ws"
    _check(st, name, check)
    return out, topk_idx, topk_w


MOE_STATIC_SCRATCH_BYTES = 4 << 20


class MxBank:
    """Device tensors of one layer's mxfp4 bank: gate/up q [E, inter, hidden/8] (int32, e2m1
    codes), e [E, inter, hidden/32] (uint8, e8m0 scales); down q [E, hidden, inter/8],
    e [E, hidden, inter/32]."""

    def __init__(self, wg_q, wg_e, wu_q, wu_e, wd_q, wd_e):
        self.wg_q, self.wg_e, self.wu_q, self.wu_e, self.wd_q, self.wd_e = (
            wg_q, wg_e, wu_q, wu_e, wd_q, wd_e)
        self.E, self.inter, hw = wg_q.shape
        self.hidden = hw * 8
        for name, t, shape in (("wg_e", wg_e, (self.E, self.inter, self.hidden // 32)),
                               ("wu_q", wu_q, wg_q.shape),
                               ("wu_e", wu_e, (self.E, self.inter, self.hidden // 32)),
                               ("wd_q", wd_q, (self.E, self.hidden, self.inter // 8)),
                               ("wd_e", wd_e, (self.E, self.hidden, self.inter // 32))):
            if tuple(t.shape) != tuple(shape):
                raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")

    def tensors(self):
        return dict(wg_q=self.wg_q, wg_e=self.wg_e, wu_q=self.wu_q, wu_e=self.wu_e,
                    wd_q=self.wd_q, wd_e=self.wd_e)

    def ptrs(self):
        return [_ptr(self.wg_q, _Q, "wg_q"), _ptr(self.wg_e, _U8, "wg_e"),
                _ptr(self.wu_q, _Q, "wu_q"), _ptr(self.wu_e, _U8, "wu_e"),
                _ptr(self.wd_q, _Q, "wd_q"), _ptr(self.wd_e, _U8, "wd_e")]


def moe_workspace_size_mxfp4(T: int, k: int, E: int, hidden: int, inter: int) -> int:
    return int(_lib.moe_workspace_size_mxfp4(T, k, E, hidden, inter))


def moe_select_path_mxfp4(T: int, k: int, E: int, hidden: int, inter: int) -> int:
    return int(_lib.moe_select_path_mxfp4(T, k, E, hidden, inter))


def _mx_args(x, topk_idx, topk_w, bank: MxBank, out):
    T, hidden = x.shape
    k = topk_idx.shape[1]
    if hidden != bank.hidden or tuple(topk_idx.shape) != (T, k) or tuple(topk_w.shape) != (T, k):
        raise ValueError("x / topk_idx / topk_w shapes do not match the bank")
    if out is None:
        out = torch.empty((T, hidden), dtype=torch.bfloat16, device=x.device)
    if tuple(out.shape) != (T, hidden):
        raise ValueError("out has the wrong shape")
    _same_device(x.device, topk_idx=topk_idx, topk_w=topk_w, out=out, **bank.tensors())
    args = [_ptr(x, _BF16, "x"), _ptr(topk_idx, _I32, "topk_idx"), _ptr(topk_w, _F32, "topk_w"),
            *bank.ptrs()]
    return args, (T, k, bank.E, hidden, bank.inter), out


def moe_switchglu_forward_mxfp4(x, topk_idx, topk_w, bank: MxBank, out=None, stream=None,
                                check: bool = True):
    """out [T, hidden] bf16 = union-of-experts SwitchGLU of x on an mxfp4 bank."""
    args, dims, out = _mx_args(x, topk_idx, topk_w, bank, out)
    with torch.cuda.device(x.device):
        st = _lib.moe_switchglu_forward_mxfp4(*args, *dims, _ptr(out, _BF16, "out"),
                                              _stream(stream, x.device))
    _check(st, "moe_switchglu_forward_mxfp4", check)
    return out


def moe_switchglu_forward_mxfp4_ws(x, topk_idx, topk_w, bank: MxBank, workspace: torch.Tensor,
                                   out=None, stream=None, check: bool = True):
    """As moe_switchglu_forward_mxfp4 with a caller-owned zeroed uint8 workspace of
    moe_workspace_size_mxfp4 bytes (same counter-region rules as moe_switchglu_forward_ws)."""
    args, dims, out = _mx_args(x, topk_idx, topk_w, bank, out)
    _same_device(x.device, workspace=workspace)
    with torch.cuda.device(x.device):
        st = _lib.moe_switchglu_forward_mxfp4_ws(*args, *dims, _ptr(out, _BF16, "out"),
                                                 _ptr(workspace, (torch.uint8,), "workspace"),
                                                 workspace.numel(), _stream(stream, x.device))
    _check(st, "moe_switchglu_forward_mxfp4_ws", check)
    return out


def moe_set_wait_limit_ns(ns: int = 0, check: bool = True) -> int:
    """Limit of the kernels' bounded waits on the current device (0: the default 2 s)."""
    return _check(_lib.moe_set_wait_limit_ns(int(ns)), "moe_set_wait_limit_ns", check)


def moe_read_device_status(stream=None) -> int:
    return int(_lib.moe_read_device_status(_stream(stream)))
