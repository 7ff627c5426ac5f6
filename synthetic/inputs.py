"""Seeded synthetic inputs for the QLoRA NF4 linear workloads.

This module only draws random numbers and casts them to the storage dtypes the
workloads use (fp32 base weights, bf16 activations and adapters).  It holds none
of the method's arithmetic: no quantization, no rounding rule of the method, no
matmul.  Both the CPU oracle (through the tests) and the CUDA path (through the
tests and the benchmark) take their inputs from here, so the two sides always
see the same bits.

Distributions (QLoRA — Fine-Tuning a 65B Model on One GPU, "Prerequisite:
LoRA's low-rank update": B is d x r, A is r x k; "NF4: sixteen levels shaped
like the weights": trained weights are roughly zero-mean normal):
  W  ~ N(0, wstd^2) fp32, shape [N, K]
  X  ~ N(0, 1) bf16, [M, K];  dY ~ N(0, 1) bf16, [M, N]
  A  ~ U(-1/sqrt(K), 1/sqrt(K)) bf16, [r, K];  B ~ N(0, 0.01^2) bf16, [N, r]

Seeds: seed(config k, linear j, role) = 1000*(k-1) + 10*j + role with role
W=0, X=1, A=2, B=3, dY=4.  CPU tensors use numpy's PCG64; tensors drawn
directly on a CUDA device use torch's Philox generator with the same seed.
"""
from __future__ import annotations

import dataclasses
import numpy as np
import torch

ROLE = {"W": 0, "X": 1, "A": 2, "B": 3, "dY": 4, "G": 5}


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    N: int  # d_out (rows of W)
    K: int  # d_in  (cols of W)


@dataclasses.dataclass(frozen=True)
class Workload:
    key: str
    index: int          # 1-based workload number, used in the seeds
    kind: str           # "linear", "mlp", "layer", "small_m"
    linears: tuple
    M: int              # tokens
    r: int
    alpha: float
    wstd: float
    Ms: tuple = ()      # small-M token counts
    codec_n: int = 0    # elements of the standalone codec tensor

    @property
    def s(self) -> float:
        return self.alpha / self.r


WORKLOADS = {
    "c1": Workload("c1", 1, "linear", (Linear("w", 256, 512),), M=16, r=8, alpha=16, wstd=0.02),
    "c2": Workload("c2", 2, "linear", (Linear("w", 4096, 4096),), M=4096, r=16, alpha=32, wstd=0.02),
    "c3": Workload("c3", 3, "mlp", (Linear("gate", 11008, 4096), Linear("up", 11008, 4096),
                                     Linear("down", 4096, 11008)), M=8192, r=64, alpha=16, wstd=0.02),
    "c4": Workload("c4", 4, "layer", (Linear("q", 8192, 8192), Linear("k", 1024, 8192),
                                       Linear("v", 1024, 8192), Linear("o", 8192, 8192),
                                       Linear("gate", 28672, 8192), Linear("up", 28672, 8192),
                                       Linear("down", 8192, 28672)), M=2048, r=16, alpha=32, wstd=0.015),
    "c5": Workload("c5", 5, "small_m", (Linear("w", 28672, 8192),), M=16, r=16, alpha=32, wstd=0.02,
                   Ms=(1, 4, 16), codec_n=4 * 2 ** 30),
}


def seed_of(index: int, j: int, role: str) -> int:
    return 1000 * (index - 1) + 10 * j + ROLE[role]


def _np_rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _torch_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, std: float, seed: int, device="cpu", dtype=torch.float32) -> torch.Tensor:
    """N(0, std^2) drawn in fp32, then cast (round-to-nearest-even) to `dtype`."""
    device = torch.device(device)
    if device.type == "cpu":
        a = _np_rng(seed).standard_normal(size=shape, dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        t = torch.from_numpy(a)
    else:
        t = torch.randn(shape, generator=_torch_gen(seed, device), device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
    return t if dtype == torch.float32 else t.to(dtype)


def uniform(shape, bound: float, seed: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """U(-bound, bound) drawn in fp32, then cast to `dtype`."""
    device = torch.device(device)
    if device.type == "cpu":
        a = _np_rng(seed).uniform(-bound, bound, size=shape).astype(np.float32)
        t = torch.from_numpy(a)
    else:
        t = torch.rand(shape, generator=_torch_gen(seed, device), device=device, dtype=torch.float32)
        t.mul_(2 * bound).sub_(bound)
    return t.to(dtype)


def linear_inputs(w: Workload, j: int, M: int | None = None, device="cpu", K_in: int | None = None):
    """W (fp32), X, A, B, dY (bf16) for linear j of workload w."""
    lin = w.linears[j]
    M = w.M if M is None else M
    K = lin.K if K_in is None else K_in
    idx = w.index
    W = normal((lin.N, lin.K), w.wstd, seed_of(idx, j, "W"), device)
    X = normal((M, K), 1.0, seed_of(idx, j, "X"), device, torch.bfloat16)
    A = uniform((w.r, lin.K), 1.0 / float(np.sqrt(lin.K)), seed_of(idx, j, "A"), device)
    B = normal((lin.N, w.r), 0.01, seed_of(idx, j, "B"), device, torch.bfloat16)
    dY = normal((M, lin.N), 1.0, seed_of(idx, j, "dY"), device, torch.bfloat16)
    return dict(W=W, X=X, A=A, B=B, dY=dY)


def codec_tensor(n: int, std: float, seed: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """A flat weight-like tensor for the standalone quantize / double-quant codec."""
    return normal((n,), std, seed, device, dtype)


def custom_weight(N: int, K: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    return normal((N, K), std, seed, device)
