"""Host-side checks of the C ABI: the library loads, exports every entry point the
header declares, and its pure host logic (path selection, workspace sizing,
argument validation before any launch) behaves as documented.  No kernel runs."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import quantized_expert_gather_b200 as qeg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_qeg.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("moe_route_union", "moe_switchglu_forward", "moe_switchglu_forward_ws",
              "moe_workspace_size", "moe_read_device_status", "moe_status_str",
              "moe_select_path", "moe_workspace_layout", "moe_switchglu_forward_static",
              "moe_router_topk", "moe_switchglu_forward_mxfp4",
              "moe_switchglu_forward_mxfp4_ws", "moe_workspace_size_mxfp4",
              "moe_select_path_mxfp4", "moe_set_wait_limit_ns", "moe_switchglu_forward_routed",
              "moe_switchglu_forward_routed_ws"):
        assert n in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", qeg.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(qeg.library_path())
    for n in declared_functions():
        assert hasattr(lib, n)


def test_status_strings():
    assert qeg.moe_status_str(0) == "MOE_OK"
    assert qeg.moe_status_str(4) == "MOE_ERR_DEVICE_INDEX"
    assert qeg.moe_status_str(99) == "MOE_ERR_UNKNOWN"


def test_path_selection_without_launch():
    # small windows -> expert-major GEMV path
    for T in (1, 2, 4, 16, 64, 128):
        assert qeg.moe_select_path(T, 8, 256, 4096, 2048) == 1
    assert qeg.moe_select_path(1024, 1, 256, 4096, 2048) == 1
    assert qeg.moe_select_path(2, 2, 16, 256, 128) == 1
    # large windows -> grouped tensor-core path (weight rows in multiples of 128)
    assert qeg.moe_select_path(512, 8, 256, 4096, 2048) == 2
    assert qeg.moe_select_path(2048, 8, 256, 4096, 2048) == 2
    assert qeg.moe_select_path(160, 8, 64, 512, 256) == 2
    assert qeg.moe_select_path(160, 8, 64, 512, 192) == 0  # inter not a multiple of 128
    # invalid shapes
    assert qeg.moe_select_path(0, 8, 256, 4096, 2048) == 0
    assert qeg.moe_select_path(4, 8, 256, 4000, 2048) == 0
    assert qeg.moe_select_path(4, 8, 256, 4096, 2000) == 0
    assert qeg.moe_select_path(4, 8, 2048, 4096, 2048) == 0  # too many experts


def test_mxfp4_path_and_workspace():
    """mxfp4 banks take the persistent kernel for small windows and the grouped path for
    large ones (GLM-5.2's 6144 x 2048 bank included); the workspace matches the affine one
    on both paths."""
    for T in (1, 2, 4, 16):
        assert qeg.moe_select_path_mxfp4(T, 8, 256, 6144, 2048) == 1
        assert qeg.moe_select_path_mxfp4(T, 8, 288, 4096, 2048) == 1
        assert qeg.moe_workspace_size_mxfp4(T, 8, 288, 4096, 2048) == \
            qeg.moe_workspace_size(T, 8, 288, 4096, 2048)
    for H in (4096, 6144):
        assert qeg.moe_select_path_mxfp4(512, 8, 256, H, 2048) == 2
        assert qeg.moe_workspace_size_mxfp4(512, 8, 256, H, 2048) == \
            qeg.moe_workspace_size(512, 8, 256, H, 2048)
    assert qeg.moe_select_path_mxfp4(160, 8, 64, 512, 192) == 0  # rows not a multiple of 128
    assert qeg.moe_workspace_size_mxfp4(0, 8, 256, 4096, 2048) == 0


def test_workspace_size_and_layout():
    T, k, E, H, I = 4, 8, 288, 4096, 2048
    n = qeg.moe_workspace_size(T, k, E, H, I)
    lay = qeg.moe_workspace_layout(T, k, E, H, I)
    assert lay["total"] == n
    assert lay["barrier"] == 0 and lay["num_unique"] >= 4 * (1 + 1024 + 512 + 2)
    # the counter region does not depend on the shape
    assert qeg.moe_workspace_layout(1, 1, 4, 64, 64)["num_unique"] == lay["num_unique"]
    assert lay["h"] % 256 == 0 and lay["h"] + 2 * T * k * I <= lay["y"]
    assert lay["y"] % 256 == 0 and lay["y"] + 4 * T * k * H <= n
    assert lay["unique"] % 16 == 0 and lay["offsets"] % 16 == 0 and lay["pair_list"] % 16 == 0
    assert qeg.moe_workspace_size(0, 8, E, H, I) == 0
    with pytest.raises(qeg.MoeError):
        qeg.moe_workspace_layout(4, 8, E, 100, I)


def test_workspace_follows_the_path():
    """The grouped path's workspace also holds the packed activations: x and h rows
    for every pair position padded to 16 per expert, bf16, and their fp32 group
    sums; the persistent kernel's does not grow with them."""
    E, H, I = 256, 4096, 2048
    for T in (512, 2048):
        P = T * 8
        assert qeg.moe_select_path(T, 8, E, H, I) == 2
        pcap = P + 15 * min(E, P)
        packed = 2 * (H + I) * pcap + 4 * (H + I) // 64 * pcap
        lay = qeg.moe_workspace_layout(T, 8, E, H, I)
        assert lay["total"] >= lay["y"] + 4 * P * H + packed
    # the small-window path stays within the 4 MiB no-allocation scratch at T=16
    assert qeg.moe_select_path(16, 8, E, H, I) == 1
    assert qeg.moe_workspace_size(16, 8, E, H, I) <= qeg.MOE_STATIC_SCRATCH_BYTES


@pytest.mark.skipif(torch.cuda.is_available(), reason="uses fake pointers; host-only check")
def test_validation_rejects_before_touching_memory():
    lib = qeg._lib
    fake = 0x10000  # never dereferenced: every call below must be rejected first
    ptrs = [fake] * 12
    # null pointer
    assert lib.moe_switchglu_forward_ws(*([None] + ptrs[1:]), 2, 2, 4, 128, 64, fake, fake,
                                        1 << 20, None) == qeg.MOE_ERR_INVALID_ARG
    # hidden not a multiple of 64
    assert lib.moe_switchglu_forward_ws(*ptrs, 2, 2, 4, 100, 64, fake, fake, 1 << 20,
                                        None) == qeg.MOE_ERR_INVALID_ARG
    # non-positive sizes
    assert lib.moe_switchglu_forward_ws(*ptrs, 0, 2, 4, 128, 64, fake, fake, 1 << 20,
                                        None) == qeg.MOE_ERR_INVALID_ARG
    # misaligned pointer
    bad = list(ptrs)
    bad[0] = fake + 2
    assert lib.moe_switchglu_forward_ws(*bad, 2, 2, 4, 128, 64, fake, fake, 1 << 20,
                                        None) == qeg.MOE_ERR_UNSUPPORTED
    # workspace too small
    assert lib.moe_switchglu_forward_ws(*ptrs, 2, 2, 4, 128, 64, fake, fake, 16,
                                        None) == qeg.MOE_ERR_WORKSPACE
    # too many experts / pairs
    assert lib.moe_switchglu_forward_ws(*ptrs, 2, 2, 5000, 128, 64, fake, fake, 1 << 20,
                                        None) == qeg.MOE_ERR_UNSUPPORTED
    assert lib.moe_route_union(fake, 70000, 1, 8, fake, fake, fake, fake,
                               None) == qeg.MOE_ERR_UNSUPPORTED
    assert lib.moe_route_union(None, 2, 2, 8, fake, fake, fake, fake,
                               None) == qeg.MOE_ERR_INVALID_ARG
    # router step: null pointers, bad sizes, k > E, limits, misalignment
    assert lib.moe_router_topk(None, 4, 16, 2, 1, fake, fake, None) == qeg.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(fake, 4, 16, 2, 1, None, fake, None) == qeg.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(fake, 0, 16, 2, 1, fake, fake, None) == qeg.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(fake, 4, 16, 17, 1, fake, fake, None) == qeg.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(fake, 4, 2048, 8, 1, fake, fake, None) == qeg.MOE_ERR_UNSUPPORTED
    assert lib.moe_router_topk(fake, 4, 64, 33, 1, fake, fake, None) == qeg.MOE_ERR_UNSUPPORTED
    assert lib.moe_router_topk(fake + 2, 4, 16, 2, 1, fake, fake, None) == qeg.MOE_ERR_UNSUPPORTED
    # router fused with the layer: null logits, k > E, E over the router's limit,
    # misaligned logits, too-small workspace
    bank = [fake] * 9
    def routed(logits, T, k, E, ws_bytes=1 << 30, out=fake, idx=fake, w=fake):
        return lib.moe_switchglu_forward_routed_ws(fake, logits, 1, *bank, T, k, E, 128, 64, out,
                                                   idx, w, fake, ws_bytes, None)
    assert routed(None, 2, 2, 4) == qeg.MOE_ERR_INVALID_ARG
    assert routed(fake, 2, 2, 4, idx=None) == qeg.MOE_ERR_INVALID_ARG
    assert routed(fake, 2, 5, 4) == qeg.MOE_ERR_INVALID_ARG
    assert routed(fake, 2, 2, 2000) == qeg.MOE_ERR_UNSUPPORTED
    assert routed(fake + 2, 2, 2, 4) == qeg.MOE_ERR_UNSUPPORTED
    assert routed(fake, 2, 2, 4, ws_bytes=16) == qeg.MOE_ERR_WORKSPACE
