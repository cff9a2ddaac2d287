"""fp64 CPU oracle for the Engram hash, gather and gate (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its Python
binding) never does, and shares no code with it.

Every function restates a definition from the page "DeepSeek 开源 TileKernels"
(zhichai.net/topic/177618722), section "5. Engram — 条件记忆门控": the n-gram
hash ``engram_hash``, the gate formula and its backward ``engram_gate_fwd/bwd``,
and the weight-gradient reduction ``engram_grad_w_reduce``.  The arithmetic lives
in ``engram_oracle.c`` (plain C, fp64); this module only marshals numpy arrays.

Gate inputs may be float64 arrays or bf16 bit patterns (``numpy.uint16``), which
are widened exactly.  Float results come back as float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "engram_oracle.c")
LIB_PATH = os.path.join(_HERE, "liboracle_engram.so")

_i64p = ctypes.POINTER(ctypes.c_int64)
_u64p = ctypes.POINTER(ctypes.c_uint64)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f64p = ctypes.POINTER(ctypes.c_double)


def build() -> str:
    """Compile the oracle library with its Makefile; returns the .so path."""
    subprocess.run(["make", "-s", "-C", _HERE], check=True)
    return LIB_PATH


def _c(a, dtype, ptype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ptype)


def _widen(a) -> np.ndarray:
    """float64 view of a gate input: bf16 bits (uint16) widen exactly."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.ascontiguousarray(a, dtype=np.float64)


class Oracle:
    """ctypes front end of one build of the oracle library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_engram_hash.argtypes = [
            _i64p, ctypes.c_int64, ctypes.c_int64, _u64p, _i32p, ctypes.c_int32,
            ctypes.c_int32, _i64p, ctypes.c_int32, ctypes.c_int64, _i64p]
        lib.oracle_engram_gather.argtypes = [
            _i64p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _i64p, _u16p,
            ctypes.c_int32, _u16p]
        lib.oracle_engram_gate_fwd.argtypes = [
            _f64p, _f64p, _f64p, _f64p, _f64p, ctypes.c_int64, ctypes.c_int32,
            ctypes.c_double, ctypes.c_double, _f64p, _f64p]
        lib.oracle_engram_gate_bwd.argtypes = [
            _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, ctypes.c_int64, ctypes.c_int32,
            ctypes.c_double, ctypes.c_double, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p]
        lib.oracle_engram_gather_bwd.argtypes = [
            _i64p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _i64p, _f64p, ctypes.c_int32,
            ctypes.c_int64, ctypes.c_int64, _f64p]
        self.lib = lib
        self.path = lib_path

    def set_threads(self, n: int) -> None:
        """OpenMP thread count the oracle uses (n <= 0 leaves it alone)."""
        self.lib.oracle_set_threads(int(n))

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def engram_hash(self, tokens, multipliers, ngram_n, table_sizes, pad_id: int = -1):
        """n-gram hash to table indices.

        tokens [B, S] int64; multipliers [L, n_max] uint64; ngram_n [L];
        table_sizes [L, J] int64.  Returns idx [B, S, L, J] int64.
        """
        tokens, tp = _c(tokens, np.int64, _i64p)
        if tokens.ndim != 2:
            raise ValueError("tokens must be [B, S]")
        B, S = tokens.shape
        mult, mp = _c(multipliers, np.uint64, _u64p)
        L, n_max = mult.shape
        nn, nnp = _c(np.asarray(ngram_n), np.int32, _i32p)
        ts, tsp = _c(table_sizes, np.int64, _i64p)
        if ts.ndim != 2 or ts.shape[0] != L or nn.shape != (L,):
            raise ValueError("shape mismatch between multipliers, ngram_n and table_sizes")
        if np.any(nn > n_max) or np.any(nn < 1) or np.any(ts < 1):
            raise ValueError("bad ngram_n or table_sizes")
        J = ts.shape[1]
        out = np.empty((B, S, L, J), dtype=np.int64)
        self.lib.oracle_engram_hash(tp, B, S, mp, nnp, L, n_max, tsp, J, int(pad_id),
                                    out.ctypes.data_as(_i64p))
        return out

    def engram_gather(self, idx, table_sizes, tables, D: int):
        """Rows idx[..., l, j] of table (l, j) from the concatenated tables.

        tables: uint16 bf16 bits holding sum(table_sizes) rows of D values.
        Returns rows [..., L, J, D] uint16.
        """
        ts, tsp = _c(table_sizes, np.int64, _i64p)
        L, J = ts.shape
        if L * J > 256:
            raise ValueError("the oracle supports at most 256 tables")
        idx = np.asarray(idx)
        lead = idx.shape[:-2]
        idx2, ip = _c(idx.reshape(-1, L, J), np.int64, _i64p)
        if np.any(idx2 < 0) or np.any(idx2 >= ts[None, :, :]):
            raise ValueError("index out of range")
        tab, tabp = _c(np.asarray(tables).reshape(-1), np.uint16, _u16p)
        if tab.size != int(ts.sum()) * D:
            raise ValueError("tables size does not match table_sizes * D")
        T = idx2.shape[0]
        out = np.empty((T, L, J, D), dtype=np.uint16)
        self.lib.oracle_engram_gather(ip, T, L, J, tsp, tabp, D, out.ctypes.data_as(_u16p))
        return out.reshape(*lead, L, J, D)

    def engram_gather_bwd(self, idx, table_sizes, d_rows, row_lo: int = 0, row_hi=None):
        """Transpose of the gather: d_rows [..., L, J, D] (float64, or bf16 bits as
        uint16) summed into the table rows they were read from.  Returns the
        global rows [row_lo, row_hi) of the concatenated tables, [rows, D] float64."""
        ts, tsp = _c(table_sizes, np.int64, _i64p)
        L, J = ts.shape
        if L * J > 256:
            raise ValueError("the oracle supports at most 256 tables")
        idx = np.asarray(idx)
        idx2, ip = _c(idx.reshape(-1, L, J), np.int64, _i64p)
        if np.any(idx2 < 0) or np.any(idx2 >= ts[None, :, :]):
            raise ValueError("index out of range")
        T = idx2.shape[0]
        dr = _widen(d_rows)
        D = dr.shape[-1]
        dr = np.ascontiguousarray(dr.reshape(T, L, J, D))
        R = int(ts.sum())
        if row_hi is None:
            row_hi = R
        if not 0 <= row_lo <= row_hi <= R:
            raise ValueError("bad row range")
        out = np.empty((row_hi - row_lo, D), dtype=np.float64)
        self.lib.oracle_engram_gather_bwd(ip, T, L, J, tsp, dr.ctypes.data_as(_f64p), D,
                                          int(row_lo), int(row_hi), out.ctypes.data_as(_f64p))
        return out

    def engram_gate_fwd(self, x, k, v, wh, we, eps: float = 1e-6, scalar: float | None = None):
        """Gate forward.  x, k, v [T, H]; wh, we [H].

        Returns (out [T, H], gate [T]) with
        gate = sigmoid(signed_sqrt(dot(RMSNorm(x, wh), RMSNorm(k, we)) * scalar)),
        out = x + gate * v and scalar = 1/sqrt(H) unless given.
        """
        x, k, v, wh, we = (_widen(a) for a in (x, k, v, wh, we))
        T, H = x.shape
        if k.shape != (T, H) or v.shape != (T, H) or wh.shape != (H,) or we.shape != (H,):
            raise ValueError("shape mismatch")
        if scalar is None:
            scalar = 1.0 / np.sqrt(float(H))
        out = np.empty((T, H), dtype=np.float64)
        gate = np.empty((T,), dtype=np.float64)
        p = lambda a: a.ctypes.data_as(_f64p)  # noqa: E731
        self.lib.oracle_engram_gate_fwd(p(x), p(k), p(v), p(wh), p(we), T, H, float(eps),
                                        float(scalar), p(out), p(gate))
        return out, gate

    def engram_gate_bwd(self, grad_out, x, k, v, wh, we, eps: float = 1e-6,
                        scalar: float | None = None, per_token: bool = True,
                        weights: bool = True):
        """Gate backward.  Returns a dict of float64 arrays: dx, dk, dv [T, H]
        (when per_token), dwh, dwe [H] summed over all T tokens (when weights),
        and the per-token statistics rx, rk, s (signed_sqrt's argument), ddot."""
        g, x, k, v, wh, we = (_widen(a) for a in (grad_out, x, k, v, wh, we))
        T, H = x.shape
        if (g.shape != (T, H) or k.shape != (T, H) or v.shape != (T, H)
                or wh.shape != (H,) or we.shape != (H,)):
            raise ValueError("shape mismatch")
        if scalar is None:
            scalar = 1.0 / np.sqrt(float(H))
        res = {}
        if per_token:
            for name in ("dx", "dk", "dv"):
                res[name] = np.empty((T, H), dtype=np.float64)
        if weights:
            res["dwh"] = np.empty((H,), dtype=np.float64)
            res["dwe"] = np.empty((H,), dtype=np.float64)
        stats = np.empty((T, 4), dtype=np.float64)
        p = lambda a: a.ctypes.data_as(_f64p)  # noqa: E731
        q = lambda name: p(res[name]) if name in res else None  # noqa: E731
        self.lib.oracle_engram_gate_bwd(p(g), p(x), p(k), p(v), p(wh), p(we), T, H,
                                        float(eps), float(scalar), q("dx"), q("dk"),
                                        q("dv"), q("dwh"), q("dwe"), p(stats))
        res.update(rx=stats[:, 0].copy(), rk=stats[:, 1].copy(), s=stats[:, 2].copy(),
                   ddot=stats[:, 3].copy())
        return res


_default: Oracle | None = None
_lock = threading.Lock()


def default() -> Oracle:
    """The oracle built from this directory's source (built on first use)."""
    global _default
    with _lock:
        if _default is None:
            if (not os.path.exists(LIB_PATH)
                    or os.path.getmtime(LIB_PATH) < os.path.getmtime(SOURCE)):
                build()
            _default = Oracle(LIB_PATH)
    return _default


def set_threads(n: int) -> None:
    default().set_threads(n)


def max_threads() -> int:
    return default().max_threads()


def engram_hash(*a, **kw):
    return default().engram_hash(*a, **kw)


def engram_gather(*a, **kw):
    return default().engram_gather(*a, **kw)


def engram_gather_bwd(*a, **kw):
    return default().engram_gather_bwd(*a, **kw)


def engram_gate_fwd(*a, **kw):
    return default().engram_gate_fwd(*a, **kw)


def engram_gate_bwd(*a, **kw):
    return default().engram_gate_bwd(*a, **kw)
