"""Helpers shared by the GPU parity tests: moving seeded host inputs to the
device and the tolerances the comparisons use.

Tolerances (the same for every test):
* hash indices and gathered rows: bit-exact;
* bf16 outputs and gradients: |gpu - ref| <= 1e-2 + 2^-8 |ref| per element,
  ref the fp64 oracle value (2^-8 |ref| bounds the final rounding to bf16);
* the fp32 gate: |gpu - ref| <= 1e-4;
* dwh, dwe: max |gpu - ref| <= 1e-3 max |ref|.
Tokens whose signed_sqrt argument is small (1e-6 <= |s| < 1e-4) amplify the
fp32 rounding of s through 1/(2 sqrt|s|); their dx/dk rows are held to 1e-2 of
the row's largest |ref| instead (see ill_conditioned()).  Below 1e-6 the
derivative's clamp makes the factor a constant, so those tokens keep the
strict bound.
"""
import numpy as np
import torch

BF16_ABS = 1e-2
BF16_REL = 2.0 ** -8
GATE_ABS = 1e-4
DW_REL = 1e-3
ILL_S = 1e-4
CLAMP_S = 1e-6


def to_dev_bf16(a: np.ndarray, dev="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_bf16_close(name, got: torch.Tensor, want: np.ndarray, rows_relaxed=None):
    g = f64(got).reshape(want.shape)
    err = np.abs(g - want)
    bound = BF16_ABS + BF16_REL * np.abs(want)
    if rows_relaxed is not None and np.any(rows_relaxed):
        rowmax = np.abs(want).max(axis=1, keepdims=True)
        bound = np.where(rows_relaxed[:, None], np.maximum(bound, 1e-2 * rowmax), bound)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{name}: {int(bad.sum())} of {err.size} elements out of tolerance; "
                             f"worst at {i}: got {g[i]!r}, want {want[i]!r}")
    return float(err.max()) if err.size else 0.0


def assert_gate_close(got: torch.Tensor, want: np.ndarray):
    err = np.abs(f64(got) - want)
    assert err.size == 0 or err.max() <= GATE_ABS, f"gate: max error {err.max()}"
    return float(err.max()) if err.size else 0.0


def assert_dw_close(name, got: torch.Tensor, want: np.ndarray):
    err = np.abs(f64(got) - want).max()
    scale = np.abs(want).max()
    assert err <= DW_REL * scale, f"{name}: max error {err} > {DW_REL} * {scale}"
    return float(err / scale)


def ill_conditioned(s_ref: np.ndarray) -> np.ndarray:
    a = np.abs(s_ref)
    return (a >= CLAMP_S) & (a < ILL_S)


def check_gate_blockwise(o, gi, res, eps, blk=2048, forward=True):
    """Compare every element of the GPU's per-token gate outputs (out, gate,
    dx, dk, dv in `res`, torch tensors [T, H] / [T]) with the oracle, computed
    block by block of `blk` tokens so that the fp64 arrays stay small.
    Returns the oracle's dwh, dwe summed over the blocks (the weight gradient
    is linear in the tokens) and s for every token."""
    T, H = gi["x"].shape
    dw = {"dwh": np.zeros(H), "dwe": np.zeros(H)}
    s_all = np.empty(T)
    for a in range(0, T, blk):
        sl = slice(a, min(T, a + blk))
        sub = {n: (arr[sl] if arr.ndim == 2 else arr) for n, arr in gi.items()}
        if forward:
            ref_out, ref_gate = o.engram_gate_fwd(sub["x"], sub["k"], sub["v"], sub["wh"],
                                                  sub["we"], eps=eps)
            assert_bf16_close("out", res["out"][sl], ref_out)
            assert_gate_close(res["gate"][sl], ref_gate)
            del ref_out
        ref = o.engram_gate_bwd(sub["g"], sub["x"], sub["k"], sub["v"], sub["wh"], sub["we"],
                                eps=eps)
        ill = ill_conditioned(ref["s"])
        assert_bf16_close("dx", res["dx"][sl], ref["dx"], rows_relaxed=ill)
        assert_bf16_close("dk", res["dk"][sl], ref["dk"], rows_relaxed=ill)
        assert_bf16_close("dv", res["dv"][sl], ref["dv"])
        dw["dwh"] += ref["dwh"]
        dw["dwe"] += ref["dwe"]
        s_all[sl] = ref["s"]
        del ref
    return dw, s_all
