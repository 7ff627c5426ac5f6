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


class GradBucket:
    """One flat buffer holding every adapter gradient of a step, so the
    data-parallel exchange is a single all-reduce (one collective launch per
    step instead of two per linear).  `view(shape)` hands out the next
    gradient tensor (dA [r, K], dB [N, r], ...) as a view into the buffer, each
    starting on a 16-byte boundary as the library requires; the library writes
    the gradients there and `allreduce()` sums them over the ranks in place."""

    def __init__(self, shapes, dtype=torch.float32, device="cpu"):
        esz = torch.tensor([], dtype=dtype).element_size()
        align = max(1, 16 // esz)
        offs, total = [], 0
        for shp in shapes:
            n = 1
            for d in shp:
                n *= int(d)
            offs.append((total, n, tuple(int(d) for d in shp)))
            total += -(-n // align) * align
        self.buffer = torch.zeros(max(total, align), dtype=dtype, device=device)
        self.views = [self.buffer[o:o + n].view(shp) for o, n, shp in offs]

    def allreduce(self, group=None) -> None:
        dist.all_reduce(self.buffer, op=dist.ReduceOp.SUM, group=group)


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor, group=None) -> None:
    """Sum dA and dB over the ranks in place (every rank gets the total), as
    one all-reduce: directly when dB follows dA in one contiguous storage (a
    GradBucket), else through one packed copy."""
    if (dA.is_contiguous() and dB.is_contiguous() and dA.dtype == dB.dtype
            and dA.untyped_storage().data_ptr() == dB.untyped_storage().data_ptr()
            and dB.data_ptr() - dA.data_ptr() == dA.numel() * dA.element_size()):
        flat = dA.new_empty(0).set_(dA.untyped_storage(), dA.storage_offset(), (dA.numel() + dB.numel(),))
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
        return
    flat = torch.cat([dA.reshape(-1), dB.reshape(-1)])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    dA.copy_(flat[:dA.numel()].view_as(dA))
    dB.copy_(flat[dA.numel():].view_as(dB))


def quantize_sharded(W_slab: torch.Tensor, group=None):
    """NF4 + double quantization of a weight split by rows over the ranks, each
    rank passing its own slab (fp32 or bf16, on its device).  Every slab but the
    last must hold a multiple of 2048 block constants (rows * cols / 64), so the
    mean's tree splits into whole level-1 nodes; the ranks all-gather their
    nodes and each finishes the tree.  Returns this slab's NF4Weight; together
    the slabs equal nf4_quantize + nf4_double_quant of the whole weight."""
    from . import _lib as L
    rows, cols = W_slab.shape
    n = rows * cols
    if n % 64:
        raise ValueError("a slab must hold whole 64-blocks")
    dev = W_slab.device
    nb = n // 64
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    L.nf4_quantize(W_slab, codes, absmax)
    nodes = torch.empty(-(-nb // 2048), dtype=torch.float64, device=dev)
    L.nf4_double_quant_level1(absmax, nodes)
    world = dist.get_world_size(group)
    # the exchange runs on the device under NCCL and through host memory under gloo
    xdev = dev if dist.get_backend(group) == "nccl" else torch.device("cpu")
    counts = [torch.zeros(1, dtype=torch.int64, device=xdev) for _ in range(world)]
    dist.all_gather(counts, torch.tensor([nb], dtype=torch.int64, device=xdev), group=group)
    nbs = [int(c.item()) for c in counts]
    if any(x % 2048 for x in nbs[:-1]):
        raise ValueError("every slab but the last must hold a multiple of 2048 block constants")
    most = max(-(-x // 2048) for x in nbs)
    mine = torch.zeros(most, dtype=torch.float64, device=xdev)
    mine[:nodes.numel()] = nodes.to(xdev)
    gathered = [torch.empty(most, dtype=torch.float64, device=xdev) for _ in range(world)]
    dist.all_gather(gathered, mine, group=group)
    all_nodes = torch.cat([g[:-(-x // 2048)] for g, x in zip(gathered, nbs)]).to(dev).contiguous()
    nb_total = sum(nbs)
    absmax_q = torch.empty(nb, dtype=torch.uint8, device=dev)
    scale2 = torch.empty(-(-nb // 256), dtype=torch.float32, device=dev)
    offset = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, L.qlora_workspace_size(L.QL_OP_DOUBLE_QUANT, nb_total)), dtype=torch.uint8, device=dev)
    L.nf4_double_quant_finish(all_nodes, nb_total, absmax, absmax_q, scale2, offset, ws)
    return L.NF4Weight(rows, cols, codes, absmax_q=absmax_q, scale2=scale2, offset=offset)
