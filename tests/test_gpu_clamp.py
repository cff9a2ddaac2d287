"""The clamp in the derivative of signed_sqrt, on the GPU.

signed_sqrt(s) = sign(s) sqrt(|s|) (page "DeepSeek 开源 TileKernels",
zhichai.net/topic/177618722, section "5. Engram — 条件记忆门控") has no finite
derivative at s = 0; the backward uses 1 / (2 sqrt(max(|s|, 1e-6))).  These
tests put tokens inside the clamp through the tuned kernels (H = 256, 4096,
7168) and the generic ones (odd H), and compare every output with the oracle
at the stated tolerances, without the relaxation for ill-conditioned tokens
(inside the clamp the derivative is a constant, so nothing is amplified):

* s = 0 exactly: x and k on disjoint columns, so every product x_j k_j is 0
  in any arithmetic and the gate is 0.5 exactly;
* 0 < |s| < 1e-6: the same, plus one shared column with x_c = +-2^-24 and
  k_c = 1, so the dot product is +-2^-24 w_c;
* ordinary N(0,1) tokens beside them.
"""
import numpy as np
import pytest
import torch

import engram_conditional_memory_hash_b200 as eng
from engram_conditional_memory_hash_b200 import inputs
from parity import (assert_bf16_close, assert_dw_close, assert_gate_close, ill_conditioned,
                    to_dev_bf16)

pytestmark = pytest.mark.gpu

CLAMP = 1e-6


def _clamp_inputs(T, H, index):
    """Gate inputs (bf16 bits) whose tokens t with t % 3 == 0 have s = 0, t % 3 == 1
    have 0 < |s| < 1e-6 and t % 3 == 2 are ordinary."""
    gi = inputs.gate_inputs(inputs.Workload("clamp", index, B=1, S=T, H=H, backward=True))
    x = inputs.bf16_bits_to_f32(gi["x"]).reshape(T, H).copy()
    k = inputs.bf16_bits_to_f32(gi["k"]).reshape(T, H).copy()
    kind = np.arange(T) % 3
    inside = kind < 2
    x[inside, 1::2] = 0.0          # x on even columns only
    k[inside, 0::2] = 0.0          # k on odd columns only
    c = 1 if H > 1 else 0
    tiny = kind == 1
    sign = np.where(np.arange(T) % 2 == 0, 1.0, -1.0).astype(np.float32)
    x[tiny, c] = sign[tiny] * np.float32(2.0 ** -24)
    k[tiny, c] = 1.0
    gi["x"] = inputs.f32_to_bf16_bits(x)
    gi["k"] = inputs.f32_to_bf16_bits(k)
    return gi, kind


@pytest.mark.parametrize("T,H", [(60, 256), (45, 4096), (33, 7168), (30, 1001), (21, 7169)])
def test_backward_inside_the_clamp(oracle_lib, T, H):
    gi, kind = _clamp_inputs(T, H, 400 + H % 13)
    t = {n: to_dev_bf16(a) for n, a in gi.items()}
    out, gate = eng.engram_gate_fwd(t["x"], t["k"], t["v"], t["wh"], t["we"])
    dx, dk, dv, part = eng.engram_gate_bwd(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"])
    dwh, dwe = eng.engram_grad_w_reduce(part, t["wh"], t["we"])
    fused = eng.engram_gate_bwd_fused(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"],
                                      G=part.shape[0])
    torch.cuda.synchronize()
    assert eng.engram_read_device_error() == 0

    ref_out, ref_gate = oracle_lib.engram_gate_fwd(gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
    ref = oracle_lib.engram_gate_bwd(gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
    s = ref["s"]
    # the planted tokens are where they should be
    assert np.all(s[kind == 0] == 0.0)
    assert np.all((np.abs(s[kind == 1]) > 0) & (np.abs(s[kind == 1]) < CLAMP / 8))

    # s = 0: the gate is 0.5 exactly, and dv = gate * g is exact in bf16
    g0 = torch.from_numpy(np.flatnonzero(kind == 0)).cuda()
    assert torch.all(gate[g0] == 0.5)
    half_g = (0.5 * t["g"][g0].float()).to(torch.bfloat16)
    assert torch.equal(dv[g0].view(torch.int16), half_g.view(torch.int16))

    relax = ill_conditioned(s)
    assert not relax[kind < 2].any()
    assert_bf16_close("out", out, ref_out)
    assert_gate_close(gate, ref_gate)
    assert_bf16_close("dx", dx, ref["dx"], rows_relaxed=relax)
    assert_bf16_close("dk", dk, ref["dk"], rows_relaxed=relax)
    assert_bf16_close("dv", dv, ref["dv"])
    assert_dw_close("dwh", dwh, ref["dwh"])
    assert_dw_close("dwe", dwe, ref["dwe"])
    for name, a, b in zip(("dx", "dk", "dv", "dwh", "dwe"), (dx, dk, dv, dwh, dwe), fused):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), "fused " + name



@pytest.mark.parametrize("T,H", [(40, 256), (24, 4096), (17, 7168), (19, 1001)])
def test_zero_fused_weight(oracle_lib, T, H):
    # wh = 0 makes the fused weight w = wh * we zero, so every token has
    # dot = 0, s = 0 and gate = 0.5 exactly; then out = x + v/2, and the
    # backward's dd (inside the clamp, finite) multiplies only terms that are
    # zero: dx = g and dk = 0 exactly, dv = g/2 exactly, dwe = wh * P = 0;
    # dwh = we * P is compared with the oracle
    gi = inputs.gate_inputs(inputs.Workload("zero_w", 500 + H % 11, B=1, S=T, H=H, backward=True))
    gi["wh"] = np.zeros_like(gi["wh"])
    t = {n: to_dev_bf16(a) for n, a in gi.items()}
    out, gate = eng.engram_gate_fwd(t["x"], t["k"], t["v"], t["wh"], t["we"])
    dx, dk, dv, dwh, dwe = eng.engram_gate_bwd_fused(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"])
    torch.cuda.synchronize()
    assert eng.engram_read_device_error() == 0
    assert torch.all(gate == 0.5)
    want_out = (t["x"].float() + 0.5 * t["v"].float()).to(torch.bfloat16)
    assert torch.equal(out.view(torch.int16), want_out.view(torch.int16))
    assert torch.equal(dx.view(torch.int16), t["g"].view(torch.int16))
    assert torch.all(dk.float() == 0.0)
    assert torch.equal(dv.view(torch.int16), (0.5 * t["g"].float()).to(torch.bfloat16).view(torch.int16))
    assert torch.all(dwe == 0.0)
    ref = oracle_lib.engram_gate_bwd(gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
    assert np.all(ref["s"] == 0.0)
    assert_dw_close("dwh", dwh, ref["dwh"])
    assert np.abs(ref["dwh"]).max() > 0       # the reduced gradient is not trivially zero
