"""The C-ABI library without a GPU: it loads, exports every symbol that
include/engram.h declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

import engram_conditional_memory_hash_b200 as eng

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "engram.h")

OK, INVALID, UNSUPPORTED, CUDA_ERR = 0, 1, 2, 3


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"ENGRAM_API\s+[^;(]*?\b(engram_\w+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_symbols()
    for n in ("engram_hash_gather", "engram_gate_fwd", "engram_gate_bwd",
              "engram_gate_bwd_num_partials", "engram_grad_w_reduce"):
        assert n in names
    assert sorted(eng.EXPORTED) == names


def test_library_exports_every_declared_symbol():
    L = eng.lib()
    for n in declared_symbols():
        assert hasattr(L, n), n
    assert eng.engram_abi_version() == 1


def test_status_strings():
    L = eng.lib()
    for code in (OK, INVALID, UNSUPPORTED, CUDA_ERR, 99):
        assert L.engram_status_string(code)


def _fwd(L, T=4, H=64, ptr=16, out=16, eps=1e-6, scalar=0.125):
    p = ctypes.c_void_p(ptr) if ptr is not None else None
    o = ctypes.c_void_p(out) if out is not None else None
    return L.engram_gate_fwd(p, p, p, p, p, T, H, eps, scalar, o, None, None)


def test_gate_fwd_rejects_before_launch():
    L = eng.lib()
    assert _fwd(L, H=0) == UNSUPPORTED
    assert _fwd(L, H=65544) == UNSUPPORTED        # beyond the supported range
    assert b"not in [1, 65536]" in L.engram_last_error()
    assert _fwd(L, T=-1) == INVALID
    assert _fwd(L, ptr=None) == INVALID
    assert _fwd(L, out=None) == INVALID
    assert _fwd(L, ptr=25) == INVALID               # bf16 at an odd address
    assert b"aligned" in L.engram_last_error()
    assert _fwd(L, eps=float("nan")) == INVALID
    assert _fwd(L, eps=-1.0) == INVALID
    assert _fwd(L, scalar=float("inf")) == INVALID
    assert _fwd(L, T=0) == OK                       # empty: nothing to launch


def test_gate_bwd_rejects_before_launch():
    L = eng.lib()
    p = ctypes.c_void_p(16)

    def bwd(G=1, H=64, ptr=p, part=p):
        return L.engram_gate_bwd(p, p, p, p, p, p, 4, H, 1e-6, 0.125, ptr, p, p, part, G, None)

    assert bwd(G=0) == INVALID
    assert bwd(G=2**31) == INVALID
    assert bwd(H=0) == UNSUPPORTED and bwd(H=70000) == UNSUPPORTED
    assert bwd(ptr=None) == INVALID
    assert bwd(ptr=ctypes.c_void_p(17)) == INVALID                  # bf16 at an odd address
    assert bwd(part=ctypes.c_void_p(18)) == INVALID                 # fp32 partials not 4-aligned


def test_gate_bwd_fused_rejects_before_launch():
    L = eng.lib()
    p = ctypes.c_void_p(16)

    def fused(G=1, H=64, ptr=p, part=p, tickets=p, dwh=p, dwe=p, T=4):
        return L.engram_gate_bwd_fused(p, p, p, p, p, p, T, H, 1e-6, 0.125, ptr, p, p, part, G,
                                       tickets, dwh, dwe, None)

    assert fused(G=0) == INVALID
    assert fused(G=2**31) == INVALID
    assert fused(H=0) == UNSUPPORTED and fused(H=70000) == UNSUPPORTED
    assert fused(ptr=None) == INVALID
    assert fused(tickets=None) == INVALID
    assert b"tickets" in L.engram_last_error()
    assert fused(dwh=None) == INVALID and fused(dwe=None) == INVALID
    assert fused(tickets=ctypes.c_void_p(18)) == INVALID             # tickets not 4-aligned
    assert fused(dwe=ctypes.c_void_p(18)) == INVALID
    assert fused(part=ctypes.c_void_p(18)) == INVALID
    assert fused(T=-1) == INVALID


def test_gate_bwd_noalloc_rejects_before_launch():
    L = eng.lib()
    p = ctypes.c_void_p(16)

    def noalloc(H=64, T=4, dwh=p):
        return L.engram_gate_bwd_noalloc(p, p, p, p, p, p, T, H, 1e-6, 0.125, p, p, p, dwh, p,
                                         None)

    # H beyond the gate's limit is refused before any device query or launch
    assert noalloc(H=65544) == UNSUPPORTED
    assert noalloc(H=0) == UNSUPPORTED
    assert noalloc(T=-1) == INVALID
    assert noalloc(dwh=None) == INVALID


def test_grad_w_reduce_rejects_before_launch():
    L = eng.lib()
    p = ctypes.c_void_p(16)
    assert L.engram_grad_w_reduce(p, 0, 64, p, p, p, p, None) == INVALID
    assert L.engram_grad_w_reduce(p, 4, 0, p, p, p, p, None) == INVALID
    assert L.engram_grad_w_reduce(None, 4, 64, p, p, p, p, None) == INVALID
    assert L.engram_grad_w_reduce(p, 4, 64, ctypes.c_void_p(17), p, p, p, None) == INVALID


def test_hash_gather_rejects_before_launch():
    import numpy as np
    L = eng.lib()
    mult = np.array([[3, 5, 0], [7, 11, 13]], dtype=np.uint64)
    nn = np.array([2, 3], dtype=np.int32)
    ts = np.full((2, 8), 4099, dtype=np.int64)
    p = ctypes.c_void_p(64)

    def hg(B=2, S=8, mult=mult, nn=nn, L_=2, n_max=3, ts=ts, J=8, tab=p, D=32, idx=p, rows=p):
        return L.engram_hash_gather(p, B, S, mult.ctypes.data if mult is not None else None,
                                    nn.ctypes.data, L_, n_max, ts.ctypes.data, J, tab, D, -1,
                                    idx, rows, None)

    assert hg(B=-1) == INVALID
    assert hg(mult=None) == INVALID
    assert hg(L_=0) == UNSUPPORTED and hg(L_=5) == UNSUPPORTED
    assert hg(J=0) == UNSUPPORTED and hg(J=17) == UNSUPPORTED
    assert hg(n_max=9) == UNSUPPORTED
    assert hg(D=12) == UNSUPPORTED and hg(D=264) == UNSUPPORTED
    assert hg(idx=None, rows=None) == INVALID
    assert hg(nn=np.array([2, 4], dtype=np.int32)) == INVALID        # n > n_max
    bad = ts.copy()
    bad[1, 3] = 0
    assert hg(ts=bad) == INVALID
    assert hg(rows=ctypes.c_void_p(72)) == INVALID                   # rows not 16-aligned
    assert hg(tab=None) == INVALID
    assert hg(B=0) == OK and hg(S=0) == OK


def test_python_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    w = torch.ones(64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        eng.engram_gate_fwd(x, x, x, w, w)


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU error path")
def test_no_device_is_reported_not_hidden():
    assert eng.lib().engram_gate_bwd_num_partials(1024, 4096) == -1
    assert eng.lib().engram_last_error()


def test_gather_bwd_rejects_before_launch():
    import numpy as np
    L = eng.lib()
    ts = np.full((2, 8), 4099, dtype=np.int64)
    p = ctypes.c_void_p(64)

    def gb(T=4, L_=2, J=8, ts=ts, D=32, idx=p, rows=p, tab=p, ws=p, nbytes=1 << 30):
        return L.engram_gather_bwd(idx, T, L_, J, ts.ctypes.data if ts is not None else None,
                                   rows, D, tab, ws, nbytes, None)

    assert gb(T=-1) == INVALID
    assert gb(L_=0) == UNSUPPORTED and gb(L_=5) == UNSUPPORTED
    assert gb(J=0) == UNSUPPORTED and gb(J=17) == UNSUPPORTED
    assert gb(D=12) == UNSUPPORTED and gb(D=264) == UNSUPPORTED
    assert gb(T=2**27) == UNSUPPORTED                                  # 2^31 entries
    assert gb(ts=None) == INVALID
    bad = ts.copy()
    bad[0, 2] = 0
    assert gb(ts=bad) == INVALID
    big = np.full((2, 8), 2**28, dtype=np.int64)                       # 2^32 rows in total
    assert gb(ts=big) == UNSUPPORTED
    assert gb(idx=None) == INVALID and gb(ws=None) == INVALID
    assert gb(idx=ctypes.c_void_p(68)) == INVALID                      # idx not 8-aligned
    assert gb(rows=ctypes.c_void_p(72)) == INVALID                     # d_rows not 16-aligned
    assert gb(tab=ctypes.c_void_p(72)) == INVALID
    assert gb(nbytes=16) == INVALID                                    # workspace too small
    assert b"workspace" in L.engram_last_error()
    assert gb(T=0, idx=None, rows=None, tab=None, ws=None) == OK       # empty: nothing to launch


def test_gather_bwd_workspace_size():
    # two (key, position) arrays of 4-byte words for the list and its radix
    # passes, two fp64 partial rows per chunk of 64 list entries and two bits
    # per table row, plus the (smaller) histograms and counts
    R = 16_000_000
    n = eng.engram_gather_bwd_workspace_size(65536, 2, 8, 64, R)
    N = 65536 * 16
    core = 16 * N + 2 * (N // 64) * 64 * 8 + 2 * R // 8
    assert core <= n <= 2 * core
    assert eng.engram_gather_bwd_workspace_size(0, 2, 8, 64, R) == 0
    with pytest.raises(eng.EngramError):
        eng.engram_gather_bwd_workspace_size(4, 2, 8, 12, R)
    with pytest.raises(eng.EngramError):
        eng.engram_gather_bwd_workspace_size(4, 2, 8, 64, 2**32)
