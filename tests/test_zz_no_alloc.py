"""engram_gate_bwd_noalloc, the allocation-free backward for callers that
cannot allocate device memory: called through the C ABI with raw pointers, its
outputs must match the allocating entry points (engram_gate_bwd with a
caller-provided partial buffer, then engram_grad_w_reduce) within the parity
tolerances, on two calls in a row with different inputs (the static scratch
keeps the previous call's contents, which must not leak into the next).

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import numpy as np
import pytest
import torch

import engram_conditional_memory_hash_b200 as eng
from engram_conditional_memory_hash_b200 import inputs
from parity import BF16_ABS, BF16_REL, DW_REL, f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def _inputs(index, T, H):
    w = inputs.Workload("noalloc", index, B=1, S=T, H=H, backward=True)
    return {n: to_dev_bf16(a) for n, a in inputs.gate_inputs(w).items()}


def _noalloc_via_abi(t, T, H):
    dx, dk, dv = (torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    dwh, dwe = (torch.empty((H,), dtype=torch.float32, device="cuda") for _ in range(2))
    st = eng.lib().engram_gate_bwd_noalloc(
        t["g"].data_ptr(), t["x"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
        t["wh"].data_ptr(), t["we"].data_ptr(), T, H, 1e-6, eng.default_scalar(H),
        dx.data_ptr(), dk.data_ptr(), dv.data_ptr(), dwh.data_ptr(), dwe.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == 0, eng.lib().engram_last_error()
    return dx, dk, dv, dwh, dwe


def _allocating(t):
    dx, dk, dv, part = eng.engram_gate_bwd(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"])
    dwh, dwe = eng.engram_grad_w_reduce(part, t["wh"], t["we"])
    return dx, dk, dv, dwh, dwe


# (1500, 2049) and (300, 16384) run the generic kernels, whose recommended
# partial-row count would not fit in the static scratch: the call lowers it
@pytest.mark.parametrize("T,H", [(2048, 7168), (333, 4096), (1500, 2049), (300, 16384)])
def test_noalloc_matches_allocating_entry_points(T, H):
    for call, index in enumerate((200, 201)):          # two calls in a row
        t = _inputs(index + H % 7, T, H)
        got = _noalloc_via_abi(t, T, H)
        want = _allocating(t)
        torch.cuda.synchronize()
        for name, a, b in zip(("dx", "dk", "dv"), got[:3], want[:3]):
            ga, wb = f64(a), f64(b)
            bad = np.abs(ga - wb) > BF16_ABS + BF16_REL * np.abs(wb)
            assert not bad.any(), f"call {call}: {name} differs in {int(bad.sum())} elements"
        for name, a, b in zip(("dwh", "dwe"), got[3:], want[3:]):
            ga, wb = f64(a), f64(b)
            assert np.abs(ga - wb).max() <= DW_REL * np.abs(wb).max(), f"call {call}: {name}"
    assert eng.engram_read_device_error() == 0


def test_noalloc_rejects_oversize_hidden_size():
    # one row of H > 65536 values: refused with a status, nothing launched
    t = _inputs(220, 2, 64)
    st = eng.lib().engram_gate_bwd_noalloc(
        t["g"].data_ptr(), t["x"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
        t["wh"].data_ptr(), t["we"].data_ptr(), 1, 65544, 1e-6, 0.125, t["x"].data_ptr(),
        t["k"].data_ptr(), t["v"].data_ptr(), t["x"].data_ptr(), t["k"].data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st in (1, 2)
    torch.cuda.synchronize()
    assert eng.engram_read_device_error() == 0


def test_noalloc_rejects_bad_arguments():
    H = 64
    t = _inputs(210, 4, H)
    with pytest.raises(eng.EngramError):
        eng.engram_gate_bwd_noalloc(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"],
                                    scalar=float("nan"))
    st = eng.lib().engram_gate_bwd_noalloc(
        t["g"].data_ptr(), t["x"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
        t["wh"].data_ptr(), t["we"].data_ptr(), 4, H, 1e-6, 0.125, t["x"].data_ptr(),
        t["k"].data_ptr(), t["v"].data_ptr(), None, None, None)
    assert st == 1
