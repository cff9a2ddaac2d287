"""PyTorch autograd integration of the fused Engram gate.

The Engram section of the page "DeepSeek 开源 TileKernels" (zhichai.net/topic/177618722,
"5. Engram — 条件记忆门控") and the page's overview describe a
``torch.autograd.Function`` wrapper around the gate kernels with forward,
backward and weight-gradient reduction.  ``EngramGateFunction`` is that wrapper
over this library's C ABI: forward = engram_gate_fwd; backward =
engram_gate_bwd followed by engram_grad_w_reduce.  ``EngramGate`` is an
``nn.Module`` holding the two RMSNorm weights.

Inputs may have any leading shape ``[..., H]``; they are viewed as ``[T, H]``.
The gate value is returned as a non-differentiable output.
"""
from __future__ import annotations

import torch

from . import default_scalar, engram_gate_bwd, engram_gate_fwd, engram_grad_w_reduce


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
        dx, dk, dv, part = engram_gate_bwd(g, x2, k2, v2, wh.contiguous(), we.contiguous(),
                                           ctx.eps, ctx.scalar)
        dwh, dwe = engram_grad_w_reduce(part, wh.contiguous(), we.contiguous())
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
