"""Double quantization of a weight quantized in row slabs (the data-parallel
path's sharded form), on one GPU: two slabs emulated by sequential calls (no
kernel waits on another), their level-1 nodes concatenated in slab order, each
slab finished with all nodes.  The concatenated codes, scales and mean equal
nf4_quantize + nf4_double_quant of the whole weight bit for bit."""
import numpy as np
import pytest
import torch

from synthetic import inputs as S

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,split", [(128, 64), (100, 64), (64, 32), (2048, 1536)])
def test_slabs_equal_the_whole(rows, split):
    import bit_nf4_quantized_10_b200 as q
    dev = "cuda"
    K = 4096                                   # 64 constants per row: 32 rows per 2048
    W = S.custom_weight(rows, K, 0.02, 5).to(dev)
    whole = q.quantize_weight(W, dq=True)
    slabs = [W[:split], W[split:]]
    parts = []
    for Ws in slabs:
        nb = Ws.numel() // 64
        codes = torch.empty(Ws.numel() // 2, dtype=torch.uint8, device=dev)
        absmax = torch.empty(nb, dtype=torch.float32, device=dev)
        q.nf4_quantize(Ws.contiguous(), codes, absmax)
        nodes = torch.empty(-(-nb // 2048), dtype=torch.float64, device=dev)
        q.nf4_double_quant_level1(absmax, nodes)
        parts.append((codes, absmax, nodes, nb))
    all_nodes = torch.cat([p[2] for p in parts]).contiguous()
    nb_total = rows * K // 64
    ws = torch.empty(q.qlora_workspace_size(q.QL_OP_DOUBLE_QUANT, nb_total), dtype=torch.uint8, device=dev)
    aq, s2, mu = [], [], []
    for codes, absmax, _, nb in parts:
        a = torch.empty(nb, dtype=torch.uint8, device=dev)
        s = torch.empty(-(-nb // 256), dtype=torch.float32, device=dev)
        o = torch.empty(1, dtype=torch.float32, device=dev)
        q.nf4_double_quant_finish(all_nodes, nb_total, absmax, a, s, o, ws)
        aq.append(a); s2.append(s); mu.append(o)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    assert torch.equal(torch.cat([p[0] for p in parts]), whole.codes)
    assert torch.equal(torch.cat(aq), whole.absmax_q)
    assert torch.equal(torch.cat(s2), whole.scale2)
    for o in mu:
        assert torch.equal(o.view(torch.int32), whole.offset.view(torch.int32))


def _sharded_worker(rank, world, port, rows_split):
    import os
    import torch.distributed as dist
    import bit_nf4_quantized_10_b200 as q
    from bit_nf4_quantized_10_b200.dp import quantize_sharded
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        W = S.custom_weight(rows_split[-1], 4096, 0.02, 9).to("cuda")
        r0, r1 = rows_split[rank], rows_split[rank + 1]
        part = quantize_sharded(W[r0:r1].contiguous())
        whole = q.quantize_weight(W, dq=True)
        torch.cuda.synchronize()
        assert q.qlora_get_status() == q.QL_OK
        b0, b1 = r0 * 4096 // 64, r1 * 4096 // 64
        assert torch.equal(part.codes, whole.codes[b0 * 32:b1 * 32])
        assert torch.equal(part.absmax_q, whole.absmax_q[b0:b1])
        assert torch.equal(part.scale2, whole.scale2[b0 // 256:-(-b1 // 256)])
        assert torch.equal(part.offset.view(torch.int32), whole.offset.view(torch.int32))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("rows_split", [[0, 64, 128], [0, 32, 100]])
def test_quantize_sharded_two_ranks_gloo(rows_split):
    """dp.quantize_sharded with two ranks (gloo, both on this GPU, each running
    only its own slab's kernels): every rank's codes, scales and mean are its
    slice of the single-process quantization."""
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    mp.spawn(_sharded_worker, args=(2, port, rows_split), nprocs=2, join=True)
