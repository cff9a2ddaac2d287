"""GPU parity of the fused Engram gate (forward, backward, weight-gradient
reduction) against the fp64 oracle, with the tolerances stated in parity.py.
The gate is the formula of the page "DeepSeek 开源 TileKernels"
(zhichai.net/topic/177618722), section "5. Engram — 条件记忆门控"."""
import numpy as np
import pytest
import torch

import engram_conditional_memory_hash_b200 as eng
from engram_conditional_memory_hash_b200 import inputs
from parity import (assert_bf16_close, assert_dw_close, assert_gate_close, check_gate_blockwise,
                    ill_conditioned, to_dev_bf16)

pytestmark = pytest.mark.gpu


def _dev(gi):
    return {n: to_dev_bf16(a) for n, a in gi.items()}


def _same_bits(name, a, b):
    assert torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8)), name


def _gpu_path(t, eps=1e-6, G=None):
    """Forward, backward and standalone reduction; the fused backward
    (reduction in the backward kernel's tail) must give the same bits."""
    out, gate = eng.engram_gate_fwd(t["x"], t["k"], t["v"], t["wh"], t["we"], eps=eps)
    dx, dk, dv, part = eng.engram_gate_bwd(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"],
                                           eps=eps, G=G)
    dwh, dwe = eng.engram_grad_w_reduce(part, t["wh"], t["we"])
    fused = eng.engram_gate_bwd_fused(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"], eps=eps,
                                      G=part.shape[0])
    torch.cuda.synchronize()
    for name, a, b in zip(("dx", "dk", "dv", "dwh", "dwe"), (dx, dk, dv, dwh, dwe), fused):
        _same_bits("fused " + name, a, b)
    return dict(out=out, gate=gate, dx=dx, dk=dk, dv=dv, part=part, dwh=dwh, dwe=dwe)


def _check_all(o, gi, res, eps=1e-6, rows=None):
    """Compare every output with the oracle; rows: token sample for the
    per-token outputs (None: all tokens)."""
    sel = slice(None) if rows is None else rows
    sub = {n: (a[sel] if a.ndim == 2 else a) for n, a in gi.items()}
    ref_out, ref_gate = o.engram_gate_fwd(sub["x"], sub["k"], sub["v"], sub["wh"], sub["we"], eps=eps)
    ref = o.engram_gate_bwd(sub["g"], sub["x"], sub["k"], sub["v"], sub["wh"], sub["we"], eps=eps,
                            weights=rows is None)
    ill = ill_conditioned(ref["s"])
    pick = (lambda t: t) if rows is None else (lambda t: t[torch.from_numpy(np.asarray(rows)).cuda()])
    rep = {
        "out": assert_bf16_close("out", pick(res["out"]), ref_out),
        "gate": assert_gate_close(pick(res["gate"]), ref_gate),
        "dx": assert_bf16_close("dx", pick(res["dx"]), ref["dx"], rows_relaxed=ill),
        "dk": assert_bf16_close("dk", pick(res["dk"]), ref["dk"], rows_relaxed=ill),
        "dv": assert_bf16_close("dv", pick(res["dv"]), ref["dv"]),
    }
    if rows is None:
        rep["dwh"] = assert_dw_close("dwh", res["dwh"], ref["dwh"])
        rep["dwe"] = assert_dw_close("dwe", res["dwe"], ref["dwe"])
    return rep


def test_tiny(oracle_lib):
    w = inputs.WORKLOADS["tiny"]
    gi = inputs.gate_inputs(w)
    res = _gpu_path(_dev(gi))
    _check_all(oracle_lib, gi, res)
    assert eng.engram_read_device_error() == 0


@pytest.mark.parametrize("T,H", [(1, 8), (3, 264), (149, 1000 * 8 // 8 + 8), (300, 4096),
                                 (150, 7168), (37, 8192), (5, 512), (2, 4104)])
def test_shapes_and_ragged(oracle_lib, T, H):
    w = inputs.Workload("ragged", 90 + H % 17, B=1, S=T, H=H, backward=True)
    gi = inputs.gate_inputs(w)
    res = _gpu_path(_dev(gi))
    _check_all(oracle_lib, gi, res)


@pytest.mark.parametrize("G", [1, 7, 148, 400])
def test_partial_count(oracle_lib, G):
    w = inputs.Workload("partials", 60, B=1, S=300, H=1024, backward=True)
    gi = inputs.gate_inputs(w)
    res = _gpu_path(_dev(gi), G=G)
    assert tuple(res["part"].shape) == (G, 1024)
    _check_all(oracle_lib, gi, res)
    if G > 300:   # CTAs without tokens write zero partial rows
        assert torch.count_nonzero(res["part"][300:]).item() == 0


def test_closed_forms_on_gpu():
    # x and k with disjoint supports: gate = 0.5 exactly and out = x + v/2
    H, T = 256, 64
    r = np.random.default_rng(3)
    x = r.standard_normal((T, H)).astype(np.float32)
    k = r.standard_normal((T, H)).astype(np.float32)
    x[:, 1::2] = 0
    k[:, 0::2] = 0
    v = r.standard_normal((T, H)).astype(np.float32)
    t = {n: to_dev_bf16(inputs.f32_to_bf16_bits(a)) for n, a in (("x", x), ("k", k), ("v", v))}
    ones = torch.ones(H, dtype=torch.bfloat16, device="cuda")
    out, gate = eng.engram_gate_fwd(t["x"], t["k"], t["v"], ones, ones)
    torch.cuda.synchronize()
    assert torch.all(gate == 0.5)
    ref = (t["x"].float() + 0.5 * t["v"].float()).to(torch.bfloat16)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    # v = 0: out = x bit for bit
    out0, _ = eng.engram_gate_fwd(t["x"], t["k"], torch.zeros_like(t["v"]), ones, ones)
    torch.cuda.synchronize()
    assert torch.equal(out0.view(torch.int16), t["x"].view(torch.int16))
    # k = x, wh = we = 1, eps = 0: gate = sigmoid(H^(1/4))
    xx = to_dev_bf16(inputs.normal_bf16(5, 0, (T, H)))
    _, g1 = eng.engram_gate_fwd(xx, xx, xx, ones, ones, eps=0.0)
    torch.cuda.synchronize()
    assert torch.allclose(g1.double(), torch.full_like(g1.double(), 0.98201379004), atol=2e-6)


def test_deterministic(oracle_lib):
    w = inputs.Workload("det", 70, B=1, S=500, H=7168, backward=True)
    t = _dev(inputs.gate_inputs(w))
    a = _gpu_path(t)
    b = _gpu_path(t)
    for n in ("out", "gate", "dx", "dk", "dv", "part", "dwh", "dwe"):
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n


@pytest.mark.parametrize("T,H", [(3, 1), (5, 7), (129, 100), (40, 1001), (17, 8200), (9, 16384),
                                 (3, 65536), (600, 7169), (300, 2050)])
def test_generic_hidden_sizes(oracle_lib, T, H):
    # H not a multiple of 8 or above 8192: the generic kernels; every output
    # against the oracle, and G covering more and fewer CTAs than tokens
    w = inputs.Workload("generic", 180 + H % 23, B=1, S=T, H=H, backward=True)
    gi = inputs.gate_inputs(w)
    _check_all(oracle_lib, gi, _gpu_path(_dev(gi)))
    _check_all(oracle_lib, gi, _gpu_path(_dev(gi), G=max(1, T // 2)))
    assert eng.engram_read_device_error() == 0


def test_unaligned_tensors_take_the_generic_path(oracle_lib):
    # bf16 tensors starting 2 and 8 bytes past a 16-byte boundary (H = 64):
    # the tuned kernels need 16-byte aligned rows, the generic ones do not
    T, H = 37, 64
    w = inputs.Workload("unaligned", 210, B=1, S=T, H=H, backward=True)
    gi = inputs.gate_inputs(w)
    for off in (1, 4):
        t = {}
        for n, a in gi.items():
            flat = to_dev_bf16(a).reshape(-1)
            buf = torch.zeros(flat.numel() + 8, dtype=torch.bfloat16, device="cuda")
            buf[off:off + flat.numel()] = flat
            t[n] = buf[off:off + flat.numel()].view(a.shape)
        assert t["x"].data_ptr() % 16 != 0
        _check_all(oracle_lib, gi, _gpu_path(t))


def test_bad_shapes_rejected():
    big = torch.zeros(2, 65544, dtype=torch.bfloat16, device="cuda")
    w1 = torch.ones(65544, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eng.EngramError):
        eng.engram_gate_fwd(big, big, big, w1, w1)


def test_empty_tokens():
    H = 4096
    e = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    w1 = torch.ones(H, dtype=torch.bfloat16, device="cuda")
    out, gate = eng.engram_gate_fwd(e, e, e, w1, w1)
    dx, dk, dv, part = eng.engram_gate_bwd(e, e, e, e, w1, w1, G=4)
    dwh, dwe = eng.engram_grad_w_reduce(part, w1, w1)
    torch.cuda.synchronize()
    assert out.numel() == 0 and gate.numel() == 0
    assert torch.count_nonzero(part).item() == 0 and torch.count_nonzero(dwh).item() == 0


def test_gate_fwd_full_size(oracle_lib):
    """Gate forward at T = 16384, H = 4096: every output against the oracle."""
    w = inputs.WORKLOADS["gate_fwd"]
    gi = inputs.gate_inputs(w)
    del gi["g"]
    t = _dev(gi)
    out, gate = eng.engram_gate_fwd(t["x"], t["k"], t["v"], t["wh"], t["we"], eps=w.eps)
    torch.cuda.synchronize()
    ref_out, ref_gate = oracle_lib.engram_gate_fwd(gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"],
                                                   eps=w.eps)
    assert_bf16_close("out", out, ref_out)
    assert_gate_close(gate, ref_gate)


def test_gate_fwdbwd_full_size(oracle_lib):
    """Gate forward + backward at T = 32768, H = 7168 in the benchmark's launch
    configuration: every element of every per-token output against the
    oracle (computed in blocks of tokens), weight gradients over all tokens."""
    w = inputs.WORKLOADS["gate_fwdbwd"]
    gi = inputs.gate_inputs(w)
    res = _gpu_path(_dev(gi), eps=w.eps)
    dw_ref, _ = check_gate_blockwise(oracle_lib, gi, res, w.eps)
    assert_dw_close("dwh", res["dwh"], dw_ref["dwh"])
    assert_dw_close("dwe", res["dwe"], dw_ref["dwe"])
    assert eng.engram_read_device_error() == 0


@pytest.mark.parametrize("T,H,G", [(300, 4096, 1), (300, 4096, 2), (1000, 7168, 7),
                                   (4096, 7168, None), (149, 256, 148), (50, 1024, 400),
                                   (600, 8192, 33), (77, 8, 5)])
def test_fused_backward(oracle_lib, T, H, G):
    """engram_gate_bwd_fused: the same bits as the two-launch path (inside
    _gpu_path), the oracle's values, the same bits again on a second call
    (the tickets are back at zero after each call), for G from 1 to more
    partial rows than tokens."""
    w = inputs.Workload("fused", 300 + H % 29 + (G or 0), B=1, S=T, H=H, backward=True)
    gi = inputs.gate_inputs(w)
    t = _dev(gi)
    res = _gpu_path(t, G=G)
    _check_all(oracle_lib, gi, res)
    stream = torch.cuda.current_stream()
    tickets = eng._stream_tickets(t["x"].device, stream.cuda_stream)
    assert torch.count_nonzero(tickets).item() == 0
    again = eng.engram_gate_bwd_fused(t["g"], t["x"], t["k"], t["v"], t["wh"], t["we"],
                                      G=res["part"].shape[0])
    torch.cuda.synchronize()
    for name, a in zip(("dx", "dk", "dv", "dwh", "dwe"), again):
        _same_bits("second call " + name, a, res[name])
    assert torch.count_nonzero(tickets).item() == 0
    assert eng.engram_read_device_error() == 0


def test_fused_backward_empty_and_own_tickets():
    # T = 0: zero weight gradients; a caller-owned ticket array is used and left zero
    H = 4096
    e = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    w1 = torch.ones(H, dtype=torch.bfloat16, device="cuda")
    tickets = torch.zeros(eng.GATE_BWD_TICKETS, dtype=torch.int32, device="cuda")
    dwh = torch.full((H,), 7.0, device="cuda")
    dwe = torch.full((H,), 7.0, device="cuda")
    eng.engram_gate_bwd_fused(e, e, e, e, w1, w1, G=9, tickets=tickets, dwh=dwh, dwe=dwe)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dwh).item() == 0 and torch.count_nonzero(dwe).item() == 0
    assert torch.count_nonzero(tickets).item() == 0
