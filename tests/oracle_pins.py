"""What pins the oracle to something other than itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError when
the oracle disagrees with a value or property fixed by the page "DeepSeek 开源
TileKernels" (zhichai.net/topic/177618722), section "5. Engram — 条件记忆门控"
(the n-gram hash; the gate formula with signed_sqrt and scalar = 1/sqrt(H)) or
by mathematics: hand-worked hashes, arbitrary-precision brute force, closed
forms of the gate, finite differences, an independent autograd restatement,
and invariants.  The same functions run against the real oracle
(test_oracle_*.py) and against deliberately broken copies of it
(test_oracle_mutants.py), which must each fail at least one pin.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from engram_conditional_memory_hash_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hash_handworked.json")
M64 = 1 << 64


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# hash and gather
# --------------------------------------------------------------------------

def pin_hash_handworked(o):
    g = _golden()
    idx = o.engram_hash(np.array(g["tokens"], dtype=np.int64),
                        np.array(g["multipliers"], dtype=np.uint64), g["ngram_n"],
                        np.array(g["table_sizes"], dtype=np.int64), pad_id=g["pad_id"])
    assert idx.shape == (1, 3, 2, 2)
    for case in g["cases"]:
        got = idx[0, case["s"], case["layer"]].tolist()
        assert got == case["idx"], (case, got)


def pin_hash_unsigned_modulo(o):
    # one 1-gram layer, multiplier 1, token -1: h = 2^64 - 1
    g = _golden()["unsigned_modulo"]
    idx = o.engram_hash(np.array([[-1]], dtype=np.int64), np.array([[1]], dtype=np.uint64),
                        [1], np.array([[g["P"]]], dtype=np.int64))
    assert int(idx[0, 0, 0, 0]) == g["idx"]


def pin_hash_wrapping_multiply(o):
    g = _golden()["wrapping_multiply"]
    tok = np.array([int(g["token"], 16)], dtype=np.uint64).view(np.int64).reshape(1, 1)
    idx = o.engram_hash(tok, np.array([[g["m"]]], dtype=np.uint64), [1],
                        np.array([[1000003]], dtype=np.int64))
    assert int(idx[0, 0, 0, 0]) == int(g["h"], 16) % 1000003


def bigint_hash(tokens, mult, ngram_n, sizes, pad_id):
    """Arbitrary-precision restatement used only for brute force."""
    B, S = tokens.shape
    L, J = sizes.shape
    out = np.zeros((B, S, L, J), dtype=np.int64)
    for b in range(B):
        for s in range(S):
            for l in range(L):
                h = 0
                for i in range(int(ngram_n[l])):
                    t = int(tokens[b, s - i]) if s - i >= 0 else int(pad_id)
                    h ^= ((t % M64) * int(mult[l, i])) % M64
                for j in range(J):
                    out[b, s, l, j] = h % int(sizes[l, j])
    return out


def pin_hash_bruteforce(o, seeds=(1, 2, 3)):
    for seed in seeds:
        r = np.random.default_rng(seed)
        B, S, L, J, n_max = 3, 7, 3, 5, 4
        tokens = r.integers(-(2**63), 2**63 - 1, size=(B, S), dtype=np.int64)
        tokens[0, :3] = [0, 1, 2]
        mult = r.integers(0, 2**64, size=(L, n_max), dtype=np.uint64, endpoint=False) | np.uint64(1)
        ngram_n = np.array([2, 3, 4], dtype=np.int32)
        sizes = r.integers(1, 2**62, size=(L, J), dtype=np.int64)
        sizes[0, 0] = 1
        sizes[1, 1] = 2**62 + 12345
        sizes[2, 2] = 4099
        pad = int(r.integers(-(2**63), 2**63 - 1))
        got = o.engram_hash(tokens, mult, ngram_n, sizes, pad_id=pad)
        want = bigint_hash(tokens, mult, ngram_n, sizes, pad)
        np.testing.assert_array_equal(got, want)


def pin_hash_invariants(o):
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w, with_tables=False)
    P = h["table_sizes"]
    idx = o.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"], P, pad_id=h["pad_id"])
    B, S = h["tokens"].shape
    assert idx.shape == (B, S, 2, 8)
    assert np.all(idx >= 0) and np.all(idx < P[None, None])
    assert len(set(P.ravel().tolist())) == 16
    # equal trailing n-grams give equal indices, wherever they sit
    toks = h["tokens"].copy()
    toks[1, 50:53] = toks[0, 10:13]
    toks[1, 49] = (toks[0, 9] + 1) % 1000
    idx2 = o.engram_hash(toks, h["multipliers"], h["ngram_n"], P, pad_id=h["pad_id"])
    np.testing.assert_array_equal(idx2[1, 52], idx2[0, 12])
    np.testing.assert_array_equal(idx2[1, 51, 0], idx2[0, 11, 0])
    # history never crosses a sequence boundary
    alone = o.engram_hash(toks[1:2], h["multipliers"], h["ngram_n"], P, pad_id=h["pad_id"])
    np.testing.assert_array_equal(alone[0], idx2[1])


def pin_gather_rows(o):
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w)
    r = np.random.default_rng(5)
    P = h["table_sizes"]
    idx = np.stack([r.integers(0, P[l, j], size=(2, 128)) for l in range(2) for j in range(8)],
                   axis=-1).reshape(2, 128, 2, 8)
    idx[0, 0] = P - 1
    idx[0, 1] = 0
    rows = o.engram_gather(idx, P, h["tables"], w.D)
    assert rows.shape == idx.shape + (w.D,)
    first = np.concatenate([[0], np.cumsum(P.ravel())[:-1]]).reshape(2, 8)
    np.testing.assert_array_equal(rows, h["tables"][idx + first[None, None]])


# --------------------------------------------------------------------------
# gather backward (the transpose of the gather)
# --------------------------------------------------------------------------

def pin_gather_bwd_handworked(o):
    # one layer, two tables of 3 and 2 rows (global rows 0-2 and 3-4), D = 2
    idx = np.array([[[0, 1]], [[2, 1]], [[0, 0]]], dtype=np.int64).reshape(3, 1, 2)
    sizes = np.array([[3, 2]], dtype=np.int64)
    d_rows = np.arange(1, 13, dtype=np.float64).reshape(3, 1, 2, 2)
    got = o.engram_gather_bwd(idx, sizes, d_rows)
    # row 0 <- tokens 0 and 2 of table 0; row 2 <- token 1; row 3 <- token 2 of
    # table 1; row 4 <- tokens 0 and 1 of table 1; row 1 is never read
    want = np.array([[1 + 9, 2 + 10], [0, 0], [5, 6], [11, 12], [3 + 7, 4 + 8]], dtype=np.float64)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(o.engram_gather_bwd(idx, sizes, d_rows, 2, 4), want[2:4])


def pin_gather_bwd_adjoint_and_conservation(o):
    # <gather(y), d> = <y, gather_bwd(d)> for any table values y and gradients d,
    # and the gradient mass is conserved column by column
    w = inputs.WORKLOADS["tiny"]
    h = inputs.hash_inputs(w, with_tables=False)
    P = h["table_sizes"]
    idx = o.engram_hash(h["tokens"], h["multipliers"], h["ngram_n"], P, pad_id=h["pad_id"])
    r = np.random.default_rng(17)
    D = 8
    R = int(P.sum())
    y = r.standard_normal((R, D))
    d = r.standard_normal(idx.shape + (D,))
    first = np.concatenate([[0], np.cumsum(P.ravel())[:-1]]).reshape(1, 1, 2, 8)
    gathered = y[idx + first]
    g = o.engram_gather_bwd(idx, P, d)
    assert g.shape == (R, D)
    lhs = float((gathered * d).sum())
    rhs = float((y * g).sum())
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs)), (lhs, rhs)
    np.testing.assert_allclose(g.sum(0), d.reshape(-1, D).sum(0), rtol=1e-12, atol=1e-10)
    untouched = np.ones(R, dtype=bool)
    untouched[(idx + first).ravel()] = False
    assert np.all(g[untouched] == 0.0)


# --------------------------------------------------------------------------
# gate forward
# --------------------------------------------------------------------------

def _sigmoid(u):
    return 1.0 / (1.0 + math.exp(-u))


def pin_fwd_orthogonal_gives_half(o):
    r = np.random.default_rng(11)
    T, H = 4, 64
    x = r.standard_normal((T, H))
    k = r.standard_normal((T, H))
    x[:, 1::2] = 0.0   # disjoint supports: every product x_j k_j is exactly 0
    k[:, 0::2] = 0.0
    v = r.standard_normal((T, H))
    wh = 1 + 0.1 * r.standard_normal(H)
    we = 1 + 0.1 * r.standard_normal(H)
    out, gate = o.engram_gate_fwd(x, k, v, wh, we)
    assert np.all(gate == 0.5), gate
    np.testing.assert_array_equal(out, x + 0.5 * v)


def pin_fwd_v_zero_is_identity(o):
    r = np.random.default_rng(12)
    T, H = 3, 48
    x, k = r.standard_normal((T, H)), r.standard_normal((T, H))
    out, gate = o.engram_gate_fwd(x, k, np.zeros((T, H)), np.ones(H), np.ones(H))
    np.testing.assert_array_equal(out, x)
    assert np.all((gate > 0) & (gate < 1))


# sigmoid(H^(1/4)) for k = c x, wh = we = 1, eps = 0, worked by hand:
# dot = sum (x_j rx)(c x_j rk) = H, s = H / sqrt(H) = sqrt(H), u = H^(1/4).
PARALLEL_CLOSED_FORM = {256: 0.98201379004, 4096: 0.99966464987, 7168: 0.99989910270}
ANTIPARALLEL_256 = 0.01798620996
# x = k = 1, wh = we = 1, eps = 1e-6, H = 256: s = 16 / (1 + 1e-6)
ONES_EPS_256 = 0.98201375471


def pin_fwd_parallel_closed_form(o):
    r = np.random.default_rng(13)
    for H, want in PARALLEL_CLOSED_FORM.items():
        x = r.standard_normal((2, H))
        k = x * np.array([[2.5], [0.125]])
        _, gate = o.engram_gate_fwd(x, k, r.standard_normal((2, H)), np.ones(H), np.ones(H),
                                    eps=0.0)
        assert np.allclose(gate, want, rtol=0, atol=5e-11), (H, gate, want)
    x = r.standard_normal((1, 256))
    _, gate = o.engram_gate_fwd(x, -x, x, np.ones(256), np.ones(256), eps=0.0)
    assert abs(gate[0] - ANTIPARALLEL_256) < 5e-11, gate


def pin_fwd_eps_enters_rms(o):
    H = 256
    ones = np.ones((1, H))
    _, gate = o.engram_gate_fwd(ones, ones, ones, np.ones(H), np.ones(H), eps=1e-6)
    assert abs(gate[0] - ONES_EPS_256) < 5e-11, gate


def pin_fwd_scale_invariance(o):
    r = np.random.default_rng(14)
    T, H = 5, 40
    x, k, v = (r.standard_normal((T, H)) for _ in range(3))
    wh, we = 1 + 0.1 * r.standard_normal(H), 1 + 0.1 * r.standard_normal(H)
    _, g0 = o.engram_gate_fwd(x, k, v, wh, we, eps=0.0)
    _, g1 = o.engram_gate_fwd(3.0 * x, 0.25 * k, v, wh, we, eps=0.0)
    np.testing.assert_allclose(g1, g0, rtol=1e-13, atol=0)
    # and the gate depends on the product wh*we only through each column
    _, g2 = o.engram_gate_fwd(x, k, v, wh * we, np.ones(H), eps=0.0)
    np.testing.assert_allclose(g2, g0, rtol=1e-12, atol=0)


# --------------------------------------------------------------------------
# gate backward
# --------------------------------------------------------------------------

def _random_case(seed, T=3, H=24, min_abs_s=0.05):
    r = np.random.default_rng(seed)
    while True:
        x, k, v, g = (r.standard_normal((T, H)) for _ in range(4))
        wh, we = 1 + 0.1 * r.standard_normal(H), 1 + 0.1 * r.standard_normal(H)
        d = (x / np.sqrt((x * x).mean(1, keepdims=True)) * wh
             * (k / np.sqrt((k * k).mean(1, keepdims=True)) * we)).sum(1)
        if np.all(np.abs(d) / math.sqrt(H) > min_abs_s):
            return x, k, v, g, wh, we


def pin_bwd_finite_differences(o):
    x, k, v, g, wh, we = _random_case(21)
    eps = 1e-6
    res = o.engram_gate_bwd(g, x, k, v, wh, we, eps=eps)

    def loss(x_, k_, v_, wh_, we_):
        out, _ = o.engram_gate_fwd(x_, k_, v_, wh_, we_, eps=eps)
        return float((g * out).sum())

    args = [x, k, v, wh, we]
    names = ["dx", "dk", "dv", "dwh", "dwe"]
    h = 1e-6
    for a_i, name in enumerate(names):
        base = args[a_i]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[a_i][idx] += h
            minus[a_i][idx] -= h
            fd[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        np.testing.assert_allclose(res[name], fd, rtol=1e-6, atol=1e-7, err_msg=name)


def pin_bwd_matches_autograd(o):
    import torch

    for seed in (31, 32):
        x, k, v, g, wh, we = _random_case(seed, T=6, H=64)
        eps = 1e-6
        H = x.shape[1]
        res = o.engram_gate_bwd(g, x, k, v, wh, we, eps=eps)
        tx, tk, tv, twh, twe = (torch.tensor(a, dtype=torch.float64, requires_grad=True)
                                for a in (x, k, v, wh, we))
        # the formula, restated in torch: RMSNorm both sides, dot, scale,
        # signed square root, sigmoid, residual
        nx = tx * torch.rsqrt((tx * tx).mean(-1, keepdim=True) + eps) * twh
        nk = tk * torch.rsqrt((tk * tk).mean(-1, keepdim=True) + eps) * twe
        s = (nx * nk).sum(-1) / math.sqrt(H)
        gate = torch.sigmoid(torch.sign(s) * torch.sqrt(s.abs()))
        out = tx + gate[:, None] * tv
        (out * torch.tensor(g)).sum().backward()
        for name, t in (("dx", tx), ("dk", tk), ("dv", tv), ("dwh", twh), ("dwe", twe)):
            np.testing.assert_allclose(res[name], t.grad.numpy(), rtol=1e-10, atol=1e-12,
                                       err_msg=name)


def pin_bwd_clamp_at_zero(o):
    # x and k with disjoint supports: s = 0 exactly, the derivative of
    # signed_sqrt is taken at the clamp, 1 / (2 sqrt(1e-6)) = 500
    r = np.random.default_rng(41)
    T, H = 3, 32
    x, k, v, g = (r.standard_normal((T, H)) for _ in range(4))
    x[:, 1::2] = 0.0
    k[:, 0::2] = 0.0
    wh, we = 1 + 0.1 * r.standard_normal(H), 1 + 0.1 * r.standard_normal(H)
    eps = 1e-6
    scalar = 1.0 / math.sqrt(H)
    res = o.engram_gate_bwd(g, x, k, v, wh, we, eps=eps)
    assert np.all(res["s"] == 0.0)
    rx = 1 / np.sqrt((x * x).mean(1) + eps)
    rk = 1 / np.sqrt((k * k).mean(1) + eps)
    dgate = (g * v).sum(1)
    ddot = dgate * 0.25 * 500.0 * scalar
    np.testing.assert_allclose(res["ddot"], ddot, rtol=1e-13)
    # with d = 0 the RMS terms vanish: dx = g + ddot rx rk wh we k, dk = ddot rx rk wh we x
    w = wh * we
    np.testing.assert_allclose(res["dx"], g + (ddot * rx * rk)[:, None] * w * k, rtol=1e-12,
                               atol=1e-12)
    np.testing.assert_allclose(res["dk"], (ddot * rx * rk)[:, None] * w * x, rtol=1e-12,
                               atol=1e-12)
    np.testing.assert_allclose(res["dv"], 0.5 * g, rtol=0, atol=0)


def pin_bwd_weight_grad_linear_in_tokens(o):
    x, k, v, g, wh, we = _random_case(51, T=8, H=32)
    full = o.engram_gate_bwd(g, x, k, v, wh, we)
    a = o.engram_gate_bwd(g[:3], x[:3], k[:3], v[:3], wh, we)
    b = o.engram_gate_bwd(g[3:], x[3:], k[3:], v[3:], wh, we)
    for name in ("dwh", "dwe"):
        np.testing.assert_allclose(full[name], a[name] + b[name], rtol=1e-12, atol=1e-14)
    # per-token outputs of a token do not depend on the other tokens
    for name in ("dx", "dk", "dv"):
        np.testing.assert_array_equal(full[name][:3], a[name])


def pin_thread_count_independent(o):
    w = inputs.WORKLOADS["tiny"]
    gi = inputs.gate_inputs(w, T=64)
    n = o.max_threads()
    try:
        o.set_threads(1)
        r1 = o.engram_gate_bwd(gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
        o.set_threads(max(2, n))
        r2 = o.engram_gate_bwd(gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"])
    finally:
        o.set_threads(n)
    for name in ("dx", "dk", "dv", "dwh", "dwe"):
        np.testing.assert_array_equal(r1[name], r2[name])


HASH_PINS = [pin_hash_handworked, pin_hash_unsigned_modulo, pin_hash_wrapping_multiply,
             pin_hash_bruteforce, pin_hash_invariants, pin_gather_rows,
             pin_gather_bwd_handworked, pin_gather_bwd_adjoint_and_conservation]
GATE_PINS = [pin_fwd_orthogonal_gives_half, pin_fwd_v_zero_is_identity,
             pin_fwd_parallel_closed_form, pin_fwd_eps_enters_rms, pin_fwd_scale_invariance,
             pin_bwd_finite_differences, pin_bwd_matches_autograd, pin_bwd_clamp_at_zero,
             pin_bwd_weight_grad_linear_in_tokens, pin_thread_count_independent]
ALL_PINS = HASH_PINS + GATE_PINS
