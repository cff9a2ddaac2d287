"""The autograd wrapper and module over the gate kernels: the gradients that
autograd delivers are exactly the kernels' (same calls, same launch shape), and
they agree with the fp64 oracle within the parity tolerances."""
import numpy as np
import pytest
import torch

import engram_conditional_memory_hash_b200 as eng
from engram_conditional_memory_hash_b200 import inputs
from engram_conditional_memory_hash_b200.autograd import EngramGate, engram_gate
from parity import assert_bf16_close, assert_dw_close, assert_gate_close, to_dev_bf16

pytestmark = pytest.mark.gpu


def test_function_matches_direct_calls_and_oracle(oracle_lib):
    w = inputs.Workload("autograd", 300, B=3, S=50, H=512, backward=True)
    gi = inputs.gate_inputs(w)
    t = {n: to_dev_bf16(a) for n, a in gi.items()}
    B, S, H = w.B, w.S, w.H
    x = t["x"].view(B, S, H).clone().requires_grad_()
    k = t["k"].view(B, S, H).clone().requires_grad_()
    v = t["v"].view(B, S, H).clone().requires_grad_()
    wh = t["wh"].clone().requires_grad_()
    we = t["we"].clone().requires_grad_()
    out, gate = engram_gate(x, k, v, wh, we)
    assert out.shape == (B, S, H) and gate.shape == (B, S) and not gate.requires_grad
    out.backward(t["g"].view(B, S, H))
    torch.cuda.synchronize()

    d_out, d_gate = eng.engram_gate_fwd(t["x"], t["k"], t["v"], t["wh"], t["we"])
    dx, dk, dv, part = eng.engram_gate_bwd(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"])
    dwh, dwe = eng.engram_grad_w_reduce(part, t["wh"], t["we"])
    torch.cuda.synchronize()
    for got, want in ((out, d_out), (x.grad, dx), (k.grad, dk), (v.grad, dv)):
        assert torch.equal(got.reshape(-1, H).view(torch.int16), want.view(torch.int16))
    assert torch.equal(gate.reshape(-1), d_gate)
    assert torch.equal(wh.grad.view(torch.int16), dwh.to(torch.bfloat16).view(torch.int16))
    assert torch.equal(we.grad.view(torch.int16), dwe.to(torch.bfloat16).view(torch.int16))

    ref_out, ref_gate = oracle_lib.engram_gate_fwd(gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
    ref = oracle_lib.engram_gate_bwd(gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
    assert_bf16_close("out", out.detach().reshape(-1, H), ref_out)
    assert_gate_close(gate.reshape(-1), ref_gate)
    assert_bf16_close("dx", x.grad.reshape(-1, H), ref["dx"])
    assert_bf16_close("dk", k.grad.reshape(-1, H), ref["dk"])
    assert_bf16_close("dv", v.grad.reshape(-1, H), ref["dv"])
    assert_dw_close("dwh", dwh, ref["dwh"])
    assert_dw_close("dwe", dwe, ref["dwe"])


def test_module_trains_a_step():
    torch.manual_seed(0)
    H = 256
    layer = EngramGate(H, device="cuda")
    x = torch.randn(4, 32, H, device="cuda").to(torch.bfloat16).requires_grad_()
    k = torch.randn(4, 32, H, device="cuda").to(torch.bfloat16)
    v = torch.randn(4, 32, H, device="cuda").to(torch.bfloat16)
    out = layer(x, k, v)
    loss = out.float().square().mean()
    loss.backward()
    assert layer.wh.grad is not None and torch.isfinite(layer.wh.grad.float()).all()
    assert torch.count_nonzero(layer.wh.grad).item() > 0
    assert torch.count_nonzero(x.grad).item() > 0
    assert layer.last_gate.shape == (4, 32)
    opt = torch.optim.SGD(layer.parameters(), lr=10.0)
    before = layer.wh.detach().clone()
    opt.step()
    assert not torch.equal(before, layer.wh.detach())


def test_hash_gather_function_and_module(oracle_lib):
    # the tiny workload through EngramMemory: rows equal the direct call
    # (bit-exact), the tables' gradient equals engram_gather_bwd's fp32 result
    # rounded to bf16, and that agrees with the oracle's gather backward
    from engram_conditional_memory_hash_b200.autograd import EngramMemory
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w)
    mem = EngramMemory(h["table_sizes"], w.D, h["ngram_n"], h["multipliers"], pad_id=h["pad_id"],
                       device="cuda")
    with torch.no_grad():
        mem.tables.copy_(to_dev_bf16(h["tables"]).view(-1, w.D))
    tokens = torch.from_numpy(h["tokens"]).cuda()
    rows = mem(tokens)
    d_rows = to_dev_bf16(inputs.gather_grad_inputs(w)).view(rows.shape)
    rows.backward(d_rows)
    torch.cuda.synchronize()

    idx, want_rows = eng.engram_hash_gather(tokens, h["multipliers"], h["ngram_n"],
                                            h["table_sizes"], mem.tables.detach(),
                                            pad_id=h["pad_id"])
    assert torch.equal(rows.detach().view(torch.int16), want_rows.view(torch.int16))
    d_tab = eng.engram_gather_bwd(idx, h["table_sizes"], d_rows)
    torch.cuda.synchronize()
    assert mem.tables.grad.dtype == torch.bfloat16
    assert torch.equal(mem.tables.grad.view(torch.int16), d_tab.to(torch.bfloat16).view(torch.int16))
    ref = oracle_lib.engram_gather_bwd(idx.cpu().numpy(), h["table_sizes"],
                                       inputs.gather_grad_inputs(w))
    got = mem.tables.grad.float().cpu().double().numpy()
    # bf16 rounding of an exactly summed fp32 value: within 2^-8 relative
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)
