"""The allocation-free entry point (moe_switchglu_forward_static) against the
allocating one (moe_switchglu_forward) on the same inputs, two calls in a row.

Named to be collected last, so it also runs after every other GPU test has used
the library-owned workspace; it must pass alone as well."""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_gather_b200 as qeg
from tests.gpu_util import assert_parity, bf16_to_f64, to_dev_bank, to_dev_inputs
from tests.layers import make_layer

pytestmark = pytest.mark.gpu


def _pair(L):
    bank = to_dev_bank(L)
    x, idx, w = to_dev_inputs(L)
    return bank, x, idx, w


@pytest.mark.parametrize("cfg", [
    # T, k, E, H, I: a ragged small layer, then a GLM-shaped T=4 window
    (7, 6, 40, 512, 384),
    (4, 8, 64, 4096, 2048),
])
def test_static_matches_allocating_entry_two_calls(cfg):
    T, k, E, H, I = cfg
    L = make_layer(T, k, E, H, I, seed=71 + sum(cfg), routing="uniform")
    bank, x, idx, w = _pair(L)
    ref = qeg.moe_switchglu_forward(x, idx, w, bank)
    outs = []
    for _ in range(2):  # two calls in a row: the scratch counters must come back to zero
        outs.append(qeg.moe_switchglu_forward_static(x, idx, w, bank))
    torch.cuda.synchronize()
    assert qeg.moe_read_device_status() == qeg.MOE_OK
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
    # and against the oracle
    y_ref = oracle.switchglu(L.x, L.idx, L.w, L.bank, L.E)
    assert_parity(bf16_to_f64(outs[1]), y_ref, f"static T={T} H={H}")


def test_static_alternates_with_other_shapes():
    """Shapes change between calls that share the one static array."""
    La = make_layer(3, 2, 16, 256, 128, seed=5)
    Lb = make_layer(9, 4, 30, 192, 1088, seed=6)
    A, B = _pair(La), _pair(Lb)
    ra = qeg.moe_switchglu_forward(A[1], A[2], A[3], A[0])
    rb = qeg.moe_switchglu_forward(B[1], B[2], B[3], B[0])
    for _ in range(2):
        oa = qeg.moe_switchglu_forward_static(A[1], A[2], A[3], A[0])
        ob = qeg.moe_switchglu_forward_static(B[1], B[2], B[3], B[0])
        torch.cuda.synchronize()
        assert torch.equal(oa.view(torch.int16), ra.view(torch.int16))
        assert torch.equal(ob.view(torch.int16), rb.view(torch.int16))


def test_static_rejects_shapes_beyond_its_scratch():
    T, k, E, H, I = 64, 8, 1, 4096, 2048
    need = qeg.moe_workspace_size(T, k, E, H, I)
    assert need > qeg.MOE_STATIC_SCRATCH_BYTES
    dev = "cuda"
    bank = qeg.QuantBank(
        torch.zeros((E, I, H // 8), dtype=torch.int32, device=dev),
        torch.zeros((E, I, H // 64), dtype=torch.bfloat16, device=dev),
        torch.zeros((E, I, H // 64), dtype=torch.bfloat16, device=dev),
        torch.zeros((E, I, H // 8), dtype=torch.int32, device=dev),
        torch.zeros((E, I, H // 64), dtype=torch.bfloat16, device=dev),
        torch.zeros((E, I, H // 64), dtype=torch.bfloat16, device=dev),
        torch.zeros((E, H, I // 8), dtype=torch.int32, device=dev),
        torch.zeros((E, H, I // 64), dtype=torch.bfloat16, device=dev),
        torch.zeros((E, H, I // 64), dtype=torch.bfloat16, device=dev))
    x = torch.zeros((T, H), dtype=torch.bfloat16, device=dev)
    idx = torch.zeros((T, k), dtype=torch.int32, device=dev)
    w = torch.zeros((T, k), dtype=torch.float32, device=dev)
    with pytest.raises(qeg.MoeError, match="MOE_ERR_WORKSPACE"):
        qeg.moe_switchglu_forward_static(x, idx, w, bank)
    assert "4 MiB" in qeg.moe_last_error()
