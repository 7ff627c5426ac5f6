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

from bit_nf4_quantized_10_b200.dp import token_shard, allreduce_adapter_grads
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
