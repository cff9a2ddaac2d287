"""Engram conditional-memory hot path for NVIDIA B200 (sm_100a).

Thin Python binding of the C-ABI library ``libengram_b200.so`` (declared in
``include/engram.h``): the n-gram hash with its table-row gather and the
gather's backward into the tables, and the fused Engram gate
forward/backward with the weight-gradient reduction, as
listed on the page "DeepSeek 开源 TileKernels" (zhichai.net/topic/177618722),
section "5. Engram — 条件记忆门控".

The functions carry the C names.  They only check and marshal arguments:
PyTorch provides device memory (outputs are allocated with ``torch.empty``
unless passed in) and the stream (the current stream unless one is given);
every step of the computation runs in the library's CUDA kernels.  There is
no fallback: if the library is missing or no CUDA device is present the calls
raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import numpy as np
import torch

__all__ = [
    "EngramError", "library_path", "lib", "engram_abi_version",
    "engram_hash_gather", "engram_gate_fwd", "engram_gate_bwd_num_partials",
    "engram_gate_bwd", "engram_grad_w_reduce", "engram_read_device_error",
    "engram_gate_bwd_noalloc", "engram_gather_bwd_workspace_size", "engram_gather_bwd",
    "engram_gate_bwd_fused", "GATE_BWD_TICKETS", "default_scalar",
    "DEVICE_ERR_PIPELINE_TIMEOUT", "DEVICE_ERR_INDEX_RANGE",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_NAME = "libengram_b200.so"
EXPORTED = ("engram_abi_version", "engram_status_string", "engram_last_error",
            "engram_hash_gather", "engram_gate_fwd", "engram_gate_bwd_num_partials",
            "engram_gate_bwd", "engram_grad_w_reduce", "engram_read_device_error",
            "engram_gate_bwd_noalloc", "engram_gather_bwd_workspace_size", "engram_gather_bwd",
            "engram_gate_bwd_fused")

# codes of the kernels' device error word (engram_read_device_error)
DEVICE_ERR_PIPELINE_TIMEOUT = 1
DEVICE_ERR_INDEX_RANGE = 2
# words of the ticket array of engram_gate_bwd_fused (ENGRAM_GATE_BWD_TICKETS)
GATE_BWD_TICKETS = 64


class EngramError(RuntimeError):
    """A call into the Engram library failed (carries the library's message)."""

    def __init__(self, func: str, status: int, message: str):
        super().__init__(f"{func}: status {status}: {message}")
        self.func = func
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, LIBRARY_NAME)


_lib = None
_lock = threading.Lock()

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_f32 = ctypes.c_float


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library (loaded on first use; raises if not built)."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{LIBRARY_NAME} is not built (expected at {path}); build it with "
                    "`make -C engram_conditional_memory_hash_b200/csrc` or "
                    "`python -c 'import __graft_entry__ as g; g.build()'`")
            L = ctypes.CDLL(path)
            L.engram_abi_version.restype = ctypes.c_int
            L.engram_status_string.restype = ctypes.c_char_p
            L.engram_status_string.argtypes = [ctypes.c_int]
            L.engram_last_error.restype = ctypes.c_char_p
            L.engram_hash_gather.restype = ctypes.c_int
            L.engram_hash_gather.argtypes = [_vp, _i64, _i64, _vp, _vp, _i32, _i32, _vp, _i32, _vp,
                                             _i32, _i64, _vp, _vp, _vp]
            L.engram_gate_fwd.restype = ctypes.c_int
            L.engram_gate_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i32, _f32, _f32, _vp,
                                          _vp, _vp]
            L.engram_gate_bwd_num_partials.restype = _i64
            L.engram_gate_bwd_num_partials.argtypes = [_i64, _i32]
            L.engram_gate_bwd.restype = ctypes.c_int
            L.engram_gate_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _f32, _f32,
                                          _vp, _vp, _vp, _vp, _i64, _vp]
            L.engram_gate_bwd_fused.restype = ctypes.c_int
            L.engram_gate_bwd_fused.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _f32, _f32,
                                                _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp]
            L.engram_grad_w_reduce.restype = ctypes.c_int
            L.engram_grad_w_reduce.argtypes = [_vp, _i64, _i32, _vp, _vp, _vp, _vp, _vp]
            L.engram_gate_bwd_noalloc.restype = ctypes.c_int
            L.engram_gate_bwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _f32,
                                                  _f32, _vp, _vp, _vp, _vp, _vp, _vp]
            L.engram_gather_bwd_workspace_size.restype = _i64
            L.engram_gather_bwd_workspace_size.argtypes = [_i64, _i32, _i32, _i32, _i64]
            L.engram_gather_bwd.restype = ctypes.c_int
            L.engram_gather_bwd.argtypes = [_vp, _i64, _i32, _i32, _vp, _vp, _i32, _vp, _vp,
                                            ctypes.c_size_t, _vp]
            L.engram_read_device_error.restype = ctypes.c_int
            L.engram_read_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), _i32]
            _lib = L
    return _lib


def _check(func: str, status: int) -> None:
    if status != 0:
        L = lib()
        msg = L.engram_last_error().decode(errors="replace")
        kind = L.engram_status_string(status).decode()
        raise EngramError(func, status, f"{kind}: {msg}")


def engram_abi_version() -> int:
    return int(lib().engram_abi_version())


def default_scalar(H: int) -> float:
    """scalar = 1/sqrt(hidden_size) of the gate formula."""
    return 1.0 / math.sqrt(float(H))


def _stream_ptr(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _host(a, dtype) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a).astype(dtype, copy=False))


# ----------------------------------------------------------------- hash ----

def engram_hash_gather(tokens: torch.Tensor, multipliers, ngram_n, table_sizes,
                       tables: torch.Tensor | None, pad_id: int = -1, *,
                       idx_out: torch.Tensor | None = None, rows_out: torch.Tensor | None = None,
                       want_idx: bool = True, want_rows: bool = True, stream=None):
    """n-gram hash to table indices and gather of the indexed rows.

    tokens       int64 [B, S] on the GPU.
    multipliers  host uint64 [L, n_max]; ngram_n host [L]; table_sizes host [L, J].
    tables       bf16 [sum(table_sizes), D] on the GPU (tables concatenated in
                 (layer, table) order); may be None when want_rows is False.
    Returns (idx [B, S, L, J] int64 or None, rows [B, S, L, J, D] bf16 or None).
    """
    tp = _dev(tokens, "tokens", torch.int64)
    if tokens.dim() != 2:
        raise ValueError("tokens must be [B, S]")
    B, S = tokens.shape
    mult = _host(multipliers, np.uint64)
    if mult.ndim != 2:
        raise ValueError("multipliers must be [L, n_max]")
    L, n_max = mult.shape
    nn = _host(ngram_n, np.int32).reshape(-1)
    ts = _host(table_sizes, np.int64)
    if ts.ndim != 2 or ts.shape[0] != L or nn.shape != (L,):
        raise ValueError("table_sizes must be [L, J] and ngram_n [L]")
    J = ts.shape[1]
    D = 0
    tab = 0
    if want_rows:
        if tables is None:
            raise ValueError("tables are required when want_rows")
        tab = _dev(tables, "tables", torch.bfloat16)
        if tables.dim() != 2 or tables.shape[0] != int(ts.sum()):
            raise ValueError("tables must be [sum(table_sizes), D]")
        D = tables.shape[1]
    dev = tokens.device
    if want_idx and idx_out is None:
        idx_out = torch.empty((B, S, L, J), dtype=torch.int64, device=dev)
    if want_rows and rows_out is None:
        rows_out = torch.empty((B, S, L, J, D), dtype=torch.bfloat16, device=dev)
    ip = _dev(idx_out, "idx_out", torch.int64) if want_idx else None
    rp = _dev(rows_out, "rows_out", torch.bfloat16) if want_rows else None
    if want_idx and idx_out.numel() != B * S * L * J:
        raise ValueError("idx_out has the wrong size")
    if want_rows and rows_out.numel() != B * S * L * J * D:
        raise ValueError("rows_out has the wrong size")
    st = lib().engram_hash_gather(tp, B, S, mult.ctypes.data, nn.ctypes.data, L, n_max,
                                  ts.ctypes.data, J, tab or None, D, int(pad_id), ip, rp,
                                  _stream_ptr(stream))
    _check("engram_hash_gather", st)
    return (idx_out if want_idx else None), (rows_out if want_rows else None)


def engram_gather_bwd_workspace_size(T: int, L: int, J: int, D: int, total_rows: int) -> int:
    """Bytes of device workspace engram_gather_bwd needs for T tokens, L x J tables of
    total_rows rows of D values (raises for sizes it rejects)."""
    n = int(lib().engram_gather_bwd_workspace_size(int(T), int(L), int(J), int(D),
                                                   int(total_rows)))
    if n < 0:
        _check("engram_gather_bwd_workspace_size", 2)
    return n


def engram_gather_bwd(idx: torch.Tensor, table_sizes, d_rows: torch.Tensor,
                      d_tables: torch.Tensor | None = None, *,
                      workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Backward of the row gather: d_tables[row of (t, l, j)] += d_rows[t, l, j].

    idx          int64 [..., L, J] on the GPU (as returned by engram_hash_gather).
    table_sizes  host [L, J].
    d_rows       bf16 [..., L, J, D] on the GPU, the gradient of the gathered rows
                 (one row per entry of idx, in the same order).
    d_tables     fp32 [sum(table_sizes), D] on the GPU, accumulated in place
                 (a zero tensor is allocated when None).
    workspace    uint8 tensor of at least engram_gather_bwd_workspace_size bytes
                 (allocated when None).
    Returns d_tables.
    """
    ts = _host(table_sizes, np.int64)
    if ts.ndim != 2:
        raise ValueError("table_sizes must be [L, J]")
    L, J = ts.shape
    ip = _dev(idx, "idx", torch.int64)
    rp = _dev(d_rows, "d_rows", torch.bfloat16)
    if idx.dim() < 2 or tuple(idx.shape[-2:]) != (L, J):
        raise ValueError("idx must be [..., L, J]")
    T = idx.numel() // (L * J)
    if d_rows.dim() < 3 or tuple(d_rows.shape[-3:-1]) != (L, J):
        raise ValueError("d_rows must be [..., L, J, D]")
    D = d_rows.shape[-1]
    if d_rows.numel() != T * L * J * D:
        raise ValueError("d_rows must hold one row per entry of idx")
    R = int(ts.sum())
    if d_tables is None:
        d_tables = torch.zeros((R, D), dtype=torch.float32, device=d_rows.device)
    tp = _dev(d_tables, "d_tables", torch.float32)
    if tuple(d_tables.shape) != (R, D):
        raise ValueError("d_tables must be [sum(table_sizes), D]")
    need = engram_gather_bwd_workspace_size(T, L, J, D, R)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=d_rows.device)
    wp = _dev(workspace, "workspace", torch.uint8)
    st = lib().engram_gather_bwd(ip, T, L, J, ts.ctypes.data, rp, D, tp, wp, workspace.numel(),
                                 _stream_ptr(stream))
    _check("engram_gather_bwd", st)
    return d_tables


# ----------------------------------------------------------------- gate ----

def _gate_shapes(x, k, v, wh, we):
    if x.dim() != 2:
        raise ValueError("x must be [T, H]")
    T, H = x.shape
    for name, t in (("k", k), ("v", v)):
        if tuple(t.shape) != (T, H):
            raise ValueError(f"{name} must be [T, H] like x")
    for name, t in (("wh", wh), ("we", we)):
        if tuple(t.shape) != (H,):
            raise ValueError(f"{name} must be [H]")
    return T, H


def engram_gate_fwd(x, k, v, wh, we, eps: float = 1e-6, scalar: float | None = None, *,
                    out=None, gate=None, want_gate: bool = True, stream=None):
    """Fused gate forward.  x, k, v bf16 [T, H]; wh, we bf16 [H] (all on the GPU).
    Returns (out bf16 [T, H], gate fp32 [T] or None)."""
    T, H = _gate_shapes(x, k, v, wh, we)
    ptrs = [_dev(t, n, torch.bfloat16) for t, n in ((x, "x"), (k, "k"), (v, "v"), (wh, "wh"),
                                                    (we, "we"))]
    if out is None:
        out = torch.empty_like(x)
    if want_gate and gate is None:
        gate = torch.empty((T,), dtype=torch.float32, device=x.device)
    op = _dev(out, "out", torch.bfloat16)
    gp = _dev(gate, "gate", torch.float32) if want_gate else None
    if scalar is None:
        scalar = default_scalar(H)
    st = lib().engram_gate_fwd(*ptrs, T, H, float(eps), float(scalar), op, gp, _stream_ptr(stream))
    _check("engram_gate_fwd", st)
    return out, (gate if want_gate else None)


def engram_gate_bwd_num_partials(T: int, H: int) -> int:
    """Recommended number of weight-gradient partial rows G on the current device."""
    g = int(lib().engram_gate_bwd_num_partials(int(T), int(H)))
    if g < 1:
        _check("engram_gate_bwd_num_partials", 3)
    return g


def engram_gate_bwd(grad_out, x, k, v, wh, we, eps: float = 1e-6, scalar: float | None = None, *,
                    dx=None, dk=None, dv=None, w_partial=None, G: int | None = None, stream=None):
    """Gate backward.  Returns (dx, dk, dv bf16 [T, H], w_partial fp32 [G, H])."""
    T, H = _gate_shapes(x, k, v, wh, we)
    if tuple(grad_out.shape) != (T, H):
        raise ValueError("grad_out must be [T, H]")
    ptrs = [_dev(t, n, torch.bfloat16) for t, n in ((grad_out, "grad_out"), (x, "x"), (k, "k"),
                                                    (v, "v"), (wh, "wh"), (we, "we"))]
    if w_partial is not None:
        if w_partial.dim() != 2 or w_partial.shape[1] != H:
            raise ValueError("w_partial must be [G, H]")
        if G is not None and G != w_partial.shape[0]:
            raise ValueError("G does not match w_partial")
        G = w_partial.shape[0]
    if G is None:
        G = engram_gate_bwd_num_partials(T, H)
    if w_partial is None:
        w_partial = torch.empty((G, H), dtype=torch.float32, device=x.device)
    dx = torch.empty_like(x) if dx is None else dx
    dk = torch.empty_like(x) if dk is None else dk
    dv = torch.empty_like(x) if dv is None else dv
    outs = [_dev(t, n, torch.bfloat16) for t, n in ((dx, "dx"), (dk, "dk"), (dv, "dv"))]
    pp = _dev(w_partial, "w_partial", torch.float32)
    if scalar is None:
        scalar = default_scalar(H)
    st = lib().engram_gate_bwd(*ptrs, T, H, float(eps), float(scalar), *outs, pp, int(G),
                               _stream_ptr(stream))
    _check("engram_gate_bwd", st)
    return dx, dk, dv, w_partial


_tickets = {}


def _stream_tickets(device: torch.device, stream_ptr: int) -> torch.Tensor:
    """The zeroed ticket array engram_gate_bwd_fused uses for calls on one
    stream of one device (calls in stream order may share it; the kernel
    leaves it zero)."""
    key = (device.index, stream_ptr)
    t = _tickets.get(key)
    if t is None:
        t = torch.zeros((GATE_BWD_TICKETS,), dtype=torch.int32, device=device)
        _tickets[key] = t
    return t


def engram_gate_bwd_fused(grad_out, x, k, v, wh, we, eps: float = 1e-6,
                          scalar: float | None = None, *, dx=None, dk=None, dv=None,
                          w_partial=None, G: int | None = None, tickets=None, dwh=None, dwe=None,
                          stream=None):
    """Gate backward with the weight-gradient reduction fused into its tail
    (one launch for the tuned shapes).  w_partial [G, H] fp32 is scratch;
    tickets is an int32 [GATE_BWD_TICKETS] device array that is zero before the
    call and zero after it (one per stream is kept here when None).
    Returns (dx, dk, dv bf16 [T, H], dwh, dwe fp32 [H])."""
    T, H = _gate_shapes(x, k, v, wh, we)
    if tuple(grad_out.shape) != (T, H):
        raise ValueError("grad_out must be [T, H]")
    ptrs = [_dev(t, n, torch.bfloat16) for t, n in ((grad_out, "grad_out"), (x, "x"), (k, "k"),
                                                    (v, "v"), (wh, "wh"), (we, "we"))]
    if w_partial is not None:
        if w_partial.dim() != 2 or w_partial.shape[1] != H:
            raise ValueError("w_partial must be [G, H]")
        if G is not None and G != w_partial.shape[0]:
            raise ValueError("G does not match w_partial")
        G = w_partial.shape[0]
    if G is None:
        G = engram_gate_bwd_num_partials(T, H)
    if w_partial is None:
        w_partial = torch.empty((G, H), dtype=torch.float32, device=x.device)
    sp = _stream_ptr(stream)
    if tickets is None:
        tickets = _stream_tickets(x.device, sp)
    if tickets.numel() < GATE_BWD_TICKETS:
        raise ValueError(f"tickets must hold {GATE_BWD_TICKETS} words")
    dx = torch.empty_like(x) if dx is None else dx
    dk = torch.empty_like(x) if dk is None else dk
    dv = torch.empty_like(x) if dv is None else dv
    dwh = torch.empty((H,), dtype=torch.float32, device=x.device) if dwh is None else dwh
    dwe = torch.empty((H,), dtype=torch.float32, device=x.device) if dwe is None else dwe
    outs = [_dev(t, n, torch.bfloat16) for t, n in ((dx, "dx"), (dk, "dk"), (dv, "dv"))]
    if scalar is None:
        scalar = default_scalar(H)
    st = lib().engram_gate_bwd_fused(*ptrs, T, H, float(eps), float(scalar), *outs,
                                     _dev(w_partial, "w_partial", torch.float32), int(G),
                                     _dev(tickets, "tickets", torch.int32),
                                     _dev(dwh, "dwh", torch.float32),
                                     _dev(dwe, "dwe", torch.float32), sp)
    _check("engram_gate_bwd_fused", st)
    return dx, dk, dv, dwh, dwe


def engram_grad_w_reduce(w_partial, wh, we, *, dwh=None, dwe=None, stream=None):
    """dwh = we * sum_p w_partial[p], dwe = wh * sum_p w_partial[p] (fp32 [H])."""
    if w_partial.dim() != 2:
        raise ValueError("w_partial must be [G, H]")
    G, H = w_partial.shape
    pp = _dev(w_partial, "w_partial", torch.float32)
    whp = _dev(wh, "wh", torch.bfloat16)
    wep = _dev(we, "we", torch.bfloat16)
    if tuple(wh.shape) != (H,) or tuple(we.shape) != (H,):
        raise ValueError("wh and we must be [H]")
    dwh = torch.empty((H,), dtype=torch.float32, device=w_partial.device) if dwh is None else dwh
    dwe = torch.empty((H,), dtype=torch.float32, device=w_partial.device) if dwe is None else dwe
    st = lib().engram_grad_w_reduce(pp, G, H, whp, wep, _dev(dwh, "dwh", torch.float32),
                                    _dev(dwe, "dwe", torch.float32), _stream_ptr(stream))
    _check("engram_grad_w_reduce", st)
    return dwh, dwe


def engram_gate_bwd_noalloc(grad_out, x, k, v, wh, we, eps: float = 1e-6,
                            scalar: float | None = None, *, dx=None, dk=None, dv=None, dwh=None,
                            dwe=None, stream=None):
    """engram_gate_bwd + engram_grad_w_reduce with the library's static scratch
    instead of a partial-row buffer, for callers that cannot allocate device
    memory (pass every output in to allocate nothing here either).
    Returns (dx, dk, dv bf16 [T, H], dwh, dwe fp32 [H])."""
    T, H = _gate_shapes(x, k, v, wh, we)
    if tuple(grad_out.shape) != (T, H):
        raise ValueError("grad_out must be [T, H]")
    ptrs = [_dev(t, n, torch.bfloat16) for t, n in ((grad_out, "grad_out"), (x, "x"), (k, "k"),
                                                    (v, "v"), (wh, "wh"), (we, "we"))]
    dx = torch.empty_like(x) if dx is None else dx
    dk = torch.empty_like(x) if dk is None else dk
    dv = torch.empty_like(x) if dv is None else dv
    dwh = torch.empty((H,), dtype=torch.float32, device=x.device) if dwh is None else dwh
    dwe = torch.empty((H,), dtype=torch.float32, device=x.device) if dwe is None else dwe
    outs = [_dev(t, n, torch.bfloat16) for t, n in ((dx, "dx"), (dk, "dk"), (dv, "dv"))]
    if scalar is None:
        scalar = default_scalar(H)
    st = lib().engram_gate_bwd_noalloc(*ptrs, T, H, float(eps), float(scalar), *outs,
                                       _dev(dwh, "dwh", torch.float32),
                                       _dev(dwe, "dwe", torch.float32), _stream_ptr(stream))
    _check("engram_gate_bwd_noalloc", st)
    return dx, dk, dv, dwh, dwe


def engram_read_device_error(clear: bool = True) -> int:
    """Synchronise the device and return (and by default clear) the kernels'
    error word: 0, or an OR of ENGRAM_DEVICE_ERR_* codes."""
    code = ctypes.c_uint32(0)
    st = lib().engram_read_device_error(ctypes.byref(code), 1 if clear else 0)
    _check("engram_read_device_error", st)
    return int(code.value)
