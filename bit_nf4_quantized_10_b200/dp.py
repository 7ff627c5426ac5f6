"""Data-parallel plumbing for the QLoRA linear (one process per GPU).

"QLoRA — Fine-Tuning a 65B Model on One GPU", "Where the gradients actually
go": the 4-bit base weight is frozen and only the adapter matrices A and B are
trained.  So every rank holds the same quantized weight and the same adapter,
runs the forward and backward on its own shard of the tokens, and the only
exchange is the sum of the adapter gradients dA, dB over the ranks (the
gradient of the summed loss).  dX stays with its tokens.  Host-side sequencing
only: the compute is the library's kernels; the sum is torch.distributed
(NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(m_global: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, stop) of rank's tokens; the first m_global % world
    ranks take one extra token."""
    if world < 1 or not 0 <= rank < world or m_global < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(m_global, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor, group=None) -> None:
    """Sum dA and dB over the ranks in place (every rank gets the total)."""
    dist.all_reduce(dA, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dB, op=dist.ReduceOp.SUM, group=group)
