"""Data-parallel plumbing of the Engram path (one process per GPU).

Every token's outputs depend only on its own row and, for the hash, on the two
tokens before it in the same sequence, so a batch shards over ranks by whole
sequences with no exchange.  The one exchange step is the weight gradient:
dwh and dwe are sums over all tokens, so each rank reduces its own tokens
(engram_gate_bwd + engram_grad_w_reduce) and the ranks then sum the [2, H]
result with one all-reduce (NCCL over NVLink on GPUs; any backend works).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_sequences(n_seqs: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous block [start, stop) of whole sequences owned by `rank`; the
    first n_seqs % world ranks get one sequence more."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(n_seqs, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_weight_grads(dw: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the packed weight gradients dw = [dwh; dwe] ([2, H]) over ranks, in
    place.  A no-op when torch.distributed is not initialised or has one rank."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(dw, op=dist.ReduceOp.SUM, group=group)
    return dw
