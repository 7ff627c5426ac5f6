"""The data-parallel path on CPU (gloo, world size 2): each rank runs the
oracle's forward and backward on its own token shard, the adapter gradients
are summed with the library's all-reduce helper, and the result must equal the
single-process gradients of the whole batch (the gradient of the summed loss);
dX stays per token.  Also the shard arithmetic itself."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_10_b200.dp import token_shard, allreduce_adapter_grads, GradBucket
from oracle import formats as F
from oracle import lora, nf4
from synthetic import inputs as S

N, K, M, R, SCALE = 64, 128, 13, 8, 2.0


def _case():
    W = S.custom_weight(N, K, 0.02, 11)
    X = S.normal((M, K), 1.0, 12, dtype=torch.bfloat16)
    A = S.uniform((R, K), 1.0 / np.sqrt(K), 13)
    B = S.normal((N, R), 0.01, 14, dtype=torch.bfloat16)
    dY = S.normal((M, N), 1.0, 15, dtype=torch.bfloat16)
    packed, c, _ = nf4.quantize(W)
    e, s2, mu = nf4.double_quant(c)
    What = nf4.dequant(packed, N * K, nf4.dq_constants(e, s2, mu), out="bf16").reshape(N, K)
    return What, X, A, B, dY


def _worker(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        What, X, A, B, dY = _case()
        a, b = token_shard(M, rank, world)
        _, U = lora.forward(X[a:b], What, A, B, SCALE)
        g = lora.backward(X[a:b], What, A, B, SCALE, dY[a:b], U=U)
        dA = torch.from_numpy(np.ascontiguousarray(g["dA"]))
        dB = torch.from_numpy(np.ascontiguousarray(g["dB"]))
        allreduce_adapter_grads(dA, dB)
        _, Uf = lora.forward(X, What, A, B, SCALE)
        full = lora.backward(X, What, A, B, SCALE, dY, U=Uf)
        for name, got in (("dA", dA.numpy()), ("dB", dB.numpy())):
            ref = full[name]
            err = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300)
            assert err < 1e-12, (rank, name, err)
        assert np.array_equal(g["dX"], full["dX"][a:b])
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_adapter_gradients_sum_over_token_shards_gloo():
    mp.spawn(_worker, args=(2, _free_port()), nprocs=2, join=True)


@pytest.mark.parametrize("m,world", [(0, 1), (13, 2), (4096, 8), (7, 8), (1, 3)])
def test_token_shards_partition_the_batch(m, world):
    spans = [token_shard(m, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == m
    for (a0, b0), (a1, b1) in zip(spans, spans[1:]):
        assert b0 == a1
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


# ------------------------------------------------ quantization sharded by rows
# Each rank quantizes a slab of weight rows whose block constants start on a
# multiple of 2048 (a subtree of the double-quant mean's fixed adjacent-pair
# tree).  It reduces its constants to level-1 tree nodes (one float64 sum per
# 2048 constants), the ranks all-gather the nodes in rank order, and each
# finishes the tree: the mean is the single-process mean bit for bit, so every
# rank's E4M3 codes and group scales are the matching slice of the
# single-process ones (groups of 256 never straddle a slab).
KQ = 4096                       # 64 constants per row, 32 rows per 2048 constants
CHUNK = 2048


def _quant_shard_worker(rank, world, port, n_rows, rows_split):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W = S.custom_weight(n_rows, KQ, 0.02, 21)
        r0, r1 = rows_split[rank], rows_split[rank + 1]
        _, c_r, _ = nf4.quantize(W[r0:r1])
        nodes = np.array([nf4.tree_sum_f64(c_r[i:i + CHUNK]) for i in range(0, c_r.size, CHUNK)])
        counts = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(counts, torch.tensor([nodes.size], dtype=torch.int64))
        most = max(int(c.item()) for c in counts)
        mine = torch.zeros(most, dtype=torch.float64)
        mine[:nodes.size] = torch.from_numpy(nodes)
        gathered = [torch.zeros(most, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, mine)
        all_nodes = np.concatenate([g.numpy()[:int(c.item())] for g, c in zip(gathered, counts)])
        nb_total = n_rows * KQ // 64
        mu = float(F.fl32(nf4.tree_sum_f64(all_nodes) / nb_total))
        e_r, s2_r = nf4.dq_encode(c_r, mu)
        # the single-process result
        _, c, _ = nf4.quantize(W)
        e, s2, mu_ref = nf4.double_quant(c)
        assert np.float32(mu).view(np.uint32) == np.float32(mu_ref).view(np.uint32), (rank, mu, mu_ref)
        b0, b1 = r0 * KQ // 64, r1 * KQ // 64
        assert np.array_equal(e_r, e[b0:b1])
        assert np.array_equal(s2_r, s2[b0 // 256:-(-b1 // 256)])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_rows,rows_split", [(128, [0, 64, 128]), (100, [0, 64, 100])])
def test_double_quant_sharded_by_rows_gloo(n_rows, rows_split):
    mp.spawn(_quant_shard_worker, args=(2, _free_port(), n_rows, rows_split), nprocs=2, join=True)


# ------------------------------------------- one all-reduce for every gradient
def _bucket_worker(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shapes = [(8, 24), (40, 8), (8, 136), (3, 8), (1, 1)]     # ragged sizes: views start 16-byte aligned
        bucket = GradBucket(shapes)
        for i, v in enumerate(bucket.views):
            assert v.shape == shapes[i] and v.data_ptr() % 16 == 0
            v.copy_(torch.full(shapes[i], float(rank + 1) * (i + 1)))
        bucket.allreduce()
        total = sum(r + 1 for r in range(world))
        for i, v in enumerate(bucket.views):
            assert torch.equal(v, torch.full(shapes[i], float(total * (i + 1)))), i
        # the pairwise helper: adjacent views (one collective) and separate tensors (packed copy)
        pair = GradBucket([(8, 32), (16, 8)])
        dA, dB = pair.views
        dA.fill_(rank + 1.0)
        dB.fill_(2.0 * (rank + 1))
        allreduce_adapter_grads(dA, dB)
        assert torch.all(dA == total) and torch.all(dB == 2.0 * total)
        sA, sB = torch.full((8, 32), rank + 1.0), torch.full((16, 8), 3.0 * (rank + 1))
        allreduce_adapter_grads(sA, sB)
        assert torch.all(sA == total) and torch.all(sB == 3.0 * total)
    finally:
        dist.destroy_process_group()


def test_gradient_bucket_single_allreduce_gloo():
    mp.spawn(_bucket_worker, args=(2, _free_port()), nprocs=2, join=True)
