"""One step of the Engram hot path on one device, through the C ABI.

The step is the path of the page "DeepSeek 开源 TileKernels"
(zhichai.net/topic/177618722), section "5. Engram — 条件记忆门控", in call
order:

1. engram_hash_gather: the n-gram hash of every token to its table indices,
   and the gather of the 16 indexed table rows;
2. engram_gate_fwd: the fused gate forward;
3. engram_gate_bwd_fused: the gate backward, with the reduction of the
   weight-gradient partial rows into dwh, dwe in the same kernel;
4. with more than one rank, the all-reduce (sum) of the packed [2, H] weight
   gradient, the path's one exchange step (dp.allreduce_weight_grads).

The gathered rows are an output of the step, not an input of the gate: the
page defines no projection from the rows to the gate's k and v, so k and v
are inputs of their own (as are x and the upstream gradient g).

StepBuffers holds the device tensors of one step; EngramStep.run enqueues the
calls on a stream.  Every computation runs in the library's kernels.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import GATE_BWD_TICKETS, dp, engram_gate_bwd_fused, engram_gate_bwd_num_partials
from . import engram_gate_fwd, engram_hash_gather

# names of the kernel launches of one step, in order (for per-launch events)
LAUNCHES = ("hash_gather", "gate_fwd", "gate_bwd")


@dataclasses.dataclass
class StepBuffers:
    tokens: torch.Tensor            # int64 [B, S]
    x: torch.Tensor                 # bf16 [T, H]
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor                 # upstream gradient of the gate output
    idx: torch.Tensor               # int64 [B, S, L, J]
    rows: torch.Tensor              # bf16 [B, S, L, J, D]
    out: torch.Tensor               # bf16 [T, H]
    gate: torch.Tensor              # fp32 [T]
    dx: torch.Tensor
    dk: torch.Tensor
    dv: torch.Tensor
    part: torch.Tensor              # fp32 [G, H], scratch of the weight-gradient reduction
    tickets: torch.Tensor           # int32 [GATE_BWD_TICKETS], zero between calls
    dw: torch.Tensor                # fp32 [2, H]: dwh, dwe

    INPUTS = ("tokens", "x", "k", "v", "g")
    OUTPUTS = ("idx", "rows", "out", "gate", "dx", "dk", "dv", "dw")


class EngramStep:
    """The step's fixed operands on `device`: tables [sum(table_sizes), D] bf16,
    wh, we [H] bf16, and the hash parameters (host arrays)."""

    def __init__(self, B: int, S: int, H: int, device, tables: torch.Tensor, wh: torch.Tensor,
                 we: torch.Tensor, multipliers, ngram_n, table_sizes, pad_id: int = -1,
                 eps: float = 1e-6, G: int | None = None):
        self.B, self.S, self.H = int(B), int(S), int(H)
        self.T = self.B * self.S
        self.device = torch.device(device)
        self.tables, self.wh, self.we = tables, wh, we
        self.multipliers = np.asarray(multipliers, dtype=np.uint64)
        self.ngram_n = np.asarray(ngram_n, dtype=np.int32)
        self.table_sizes = np.asarray(table_sizes, dtype=np.int64)
        self.L, self.J = self.table_sizes.shape
        self.D = int(tables.shape[1])
        self.pad_id = int(pad_id)
        self.eps = float(eps)
        self.G = int(G) if G is not None else engram_gate_bwd_num_partials(self.T, self.H)

    def buffers(self) -> StepBuffers:
        """One set of device buffers for a step (contents uninitialised, the
        tickets zero)."""
        dev, T, H = self.device, self.T, self.H

        def bf(*shape):
            return torch.empty(shape, dtype=torch.bfloat16, device=dev)

        return StepBuffers(
            tokens=torch.empty((self.B, self.S), dtype=torch.int64, device=dev),
            x=bf(T, H), k=bf(T, H), v=bf(T, H), g=bf(T, H),
            idx=torch.empty((self.B, self.S, self.L, self.J), dtype=torch.int64, device=dev),
            rows=bf(self.B, self.S, self.L, self.J, self.D),
            out=bf(T, H), gate=torch.empty((T,), dtype=torch.float32, device=dev),
            dx=bf(T, H), dk=bf(T, H), dv=bf(T, H),
            part=torch.empty((self.G, H), dtype=torch.float32, device=dev),
            tickets=torch.zeros((GATE_BWD_TICKETS,), dtype=torch.int32, device=dev),
            dw=torch.empty((2, H), dtype=torch.float32, device=dev))

    def run(self, b: StepBuffers, stream: torch.cuda.Stream, events=None, group=None) -> None:
        """Enqueue the step on `stream`.  events: optional list of
        len(LAUNCHES) + 1 CUDA events recorded around the launches.  With a
        process group of more than one rank the weight gradients are summed
        over the ranks at the end (on the same stream)."""
        def mark(i):
            if events is not None:
                events[i].record(stream)

        mark(0)
        engram_hash_gather(b.tokens, self.multipliers, self.ngram_n, self.table_sizes, self.tables,
                           pad_id=self.pad_id, idx_out=b.idx, rows_out=b.rows, stream=stream)
        mark(1)
        engram_gate_fwd(b.x, b.k, b.v, self.wh, self.we, eps=self.eps, out=b.out, gate=b.gate,
                        stream=stream)
        mark(2)
        engram_gate_bwd_fused(b.g, b.x, b.k, b.v, self.wh, self.we, eps=self.eps, dx=b.dx, dk=b.dk,
                              dv=b.dv, w_partial=b.part, tickets=b.tickets, dwh=b.dw[0],
                              dwe=b.dw[1], stream=stream)
        mark(3)
        with torch.cuda.stream(stream):
            dp.allreduce_weight_grads(b.dw, group=group)
