"""PyTorch autograd integration of the Engram hot path.

The Engram section of the page "DeepSeek 开源 TileKernels" (zhichai.net/topic/177618722,
"5. Engram — 条件记忆门控") and the page's overview describe a
``torch.autograd.Function`` wrapper around the gate kernels with forward,
backward and weight-gradient reduction.  ``EngramGateFunction`` is that wrapper
over this library's C ABI: forward = engram_gate_fwd; backward =
engram_gate_bwd_fused (the backward with engram_grad_w_reduce's reduction in
its tail, bitwise the same as the two calls).  ``EngramGate`` is an
``nn.Module`` holding the two RMSNorm weights.

``EngramHashGatherFunction`` does the same for the n-gram hash and table-row
gather: forward = engram_hash_gather, backward = engram_gather_bwd (the
gradient of the gathered rows summed into the tables; tokens get none).
``EngramMemory`` is an ``nn.Module`` holding the tables and the hash
parameters.

Gate inputs may have any leading shape ``[..., H]``; they are viewed as
``[T, H]``.  The gate value is returned as a non-differentiable output.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (default_scalar, engram_gate_bwd_fused, engram_gate_fwd, engram_gather_bwd,
               engram_hash_gather)


class EngramGateFunction(torch.autograd.Function):
    """(x, k, v, wh, we) -> (out, gate), both passes in the library's kernels."""

    @staticmethod
    def forward(ctx, x, k, v, wh, we, eps: float = 1e-6, scalar: float | None = None):
        H = x.shape[-1]
        lead = x.shape[:-1]
        x2, k2, v2 = (t.reshape(-1, H).contiguous() for t in (x, k, v))
        if scalar is None:
            scalar = default_scalar(H)
        out, gate = engram_gate_fwd(x2, k2, v2, wh.contiguous(), we.contiguous(), eps, scalar)
        ctx.save_for_backward(x2, k2, v2, wh, we)
        ctx.eps, ctx.scalar, ctx.lead = eps, scalar, lead
        out, gate = out.view(*lead, H), gate.view(lead)
        ctx.mark_non_differentiable(gate)
        return out, gate

    @staticmethod
    def backward(ctx, grad_out, grad_gate):
        x2, k2, v2, wh, we = ctx.saved_tensors
        H = x2.shape[-1]
        if grad_out is None:
            grad_out = torch.zeros_like(x2)
        g = grad_out.reshape(-1, H).to(x2.dtype).contiguous()
        dx, dk, dv, dwh, dwe = engram_gate_bwd_fused(g, x2, k2, v2, wh.contiguous(),
                                                     we.contiguous(), ctx.eps, ctx.scalar)
        lead = ctx.lead
        return (dx.view(*lead, H), dk.view(*lead, H), dv.view(*lead, H),
                dwh.to(wh.dtype), dwe.to(we.dtype), None, None)


def engram_gate(x, k, v, wh, we, eps: float = 1e-6, scalar: float | None = None):
    """Differentiable fused Engram gate: returns (out, gate)."""
    return EngramGateFunction.apply(x, k, v, wh, we, eps, scalar)


class EngramGate(torch.nn.Module):
    """The Engram gate as a module: parameters wh, we (bf16, initialised to 1).

    forward(x, k, v) -> out = x + gate * v with
    gate = sigmoid(signed_sqrt(dot(RMSNorm(x, wh), RMSNorm(k, we)) / sqrt(H)));
    ``self.last_gate`` keeps the gate values of the last call (no gradient).
    """

    def __init__(self, hidden_dim: int, eps: float = 1e-6, device=None):
        super().__init__()
        self.hidden_dim = hidden_dim
        self.eps = eps
        self.wh = torch.nn.Parameter(torch.ones(hidden_dim, dtype=torch.bfloat16, device=device))
        self.we = torch.nn.Parameter(torch.ones(hidden_dim, dtype=torch.bfloat16, device=device))
        self.last_gate = None

    def forward(self, x, k, v):
        out, gate = engram_gate(x, k, v, self.wh, self.we, self.eps)
        self.last_gate = gate
        return out


class EngramHashGatherFunction(torch.autograd.Function):
    """(tokens, tables) -> rows [B, S, L, J, D]; the gradient flows into tables.

    The backward sums the rows' gradient into an fp32 table gradient
    (engram_gather_bwd: fp64 sums in a fixed order, one rounding per row) and
    returns it in the tables' dtype."""

    @staticmethod
    def forward(ctx, tokens, tables, multipliers, ngram_n, table_sizes, pad_id: int = -1):
        idx, rows = engram_hash_gather(tokens, multipliers, ngram_n, table_sizes, tables,
                                       pad_id=pad_id)
        ctx.save_for_backward(idx)
        ctx.table_sizes = np.asarray(table_sizes, dtype=np.int64)
        ctx.table_shape, ctx.table_dtype = tables.shape, tables.dtype
        return rows

    @staticmethod
    def backward(ctx, d_rows):
        (idx,) = ctx.saved_tensors
        d_tables = torch.zeros(ctx.table_shape, dtype=torch.float32, device=idx.device)
        engram_gather_bwd(idx, ctx.table_sizes, d_rows.to(torch.bfloat16).contiguous(), d_tables)
        return None, d_tables.to(ctx.table_dtype), None, None, None, None


def engram_hash_gather_rows(tokens, tables, multipliers, ngram_n, table_sizes, pad_id: int = -1):
    """Differentiable n-gram hash + gather: rows [B, S, L, J, D] (gradient into tables)."""
    return EngramHashGatherFunction.apply(tokens, tables, multipliers, ngram_n, table_sizes,
                                          pad_id)


class EngramMemory(torch.nn.Module):
    """The Engram hash embedding tables as a module.

    table_sizes [L, J] rows per table (distinct primes keep the tables of a
    layer from repeating each other), D values per row, ngram_n [L] the n of
    each layer's n-grams (e.g. (2, 3)), multipliers [L, max n] odd 64-bit
    constants of the hash.  The tables are one bf16 parameter of
    sum(table_sizes) rows, concatenated in (layer, table) order, initialised
    N(0, init_std^2).  forward(tokens [B, S] int64) -> rows [B, S, L, J, D]."""

    def __init__(self, table_sizes, D: int, ngram_n, multipliers, pad_id: int = -1,
                 init_std: float = 1.0, device=None):
        super().__init__()
        self.table_sizes = np.asarray(table_sizes, dtype=np.int64)
        self.ngram_n = np.asarray(ngram_n, dtype=np.int32)
        self.multipliers = np.asarray(multipliers, dtype=np.uint64)
        if self.table_sizes.ndim != 2 or self.multipliers.shape[0] != self.table_sizes.shape[0]:
            raise ValueError("table_sizes must be [L, J] and multipliers [L, n_max]")
        self.pad_id = int(pad_id)
        rows = int(self.table_sizes.sum())
        t = torch.empty((rows, D), dtype=torch.bfloat16, device=device)
        torch.nn.init.normal_(t, 0.0, init_std)
        self.tables = torch.nn.Parameter(t)

    def forward(self, tokens):
        return engram_hash_gather_rows(tokens, self.tables, self.multipliers, self.ngram_n,
                                       self.table_sizes, self.pad_id)
