"""The frozen-4-bit + LoRA linear, forward and backward (oracle; tests only).

Sources:
  [P3] "QLoRA — Fine-Tuning a 65B Model on One GPU":
       "Prerequisite: LoRA's low-rank update": Delta W = B A with B in R^{d x r},
       A in R^{r x k}, h = W x + B A x, r(d + k) trainable numbers.
       "Where the gradients actually go": h = dequant(W_NF4) x + B A x in BF16;
       the chain rule runs through the dequantized W^T for the input gradient;
       W is never written; only A and B receive gradients.
       "Seeing it in code": lora_alpha scales the adapter (alpha / r).
  [P2] "QLoRA: Quantize Base Weights to 4-Bit", §3: the adapter branch
       (B @ (A @ x)) * (alpha / r) runs beside the dequantized-weight product;
       gradients go only to the BF16 adapters.

Row-vector convention (tokens are rows): X [M, K], W_hat [N, K], A [r, K],
B [N, r], Y [M, N], s = alpha / r.

All products are float64 numpy matmuls of the exact bf16 / fp32 inputs.  A
tensor is rounded to bf16 exactly where the layer hands it on as a bf16 tensor
(U = X A^T saved by the forward, V = dY B in the backward, and the MLP's g, u,
h, dh, dg, du).  Outputs (Y, dX, dA, dB) are returned unrounded.  The caller
rounds them to the output dtype under test.
"""
from __future__ import annotations

import numpy as np

from .formats import F64, bf16, fl32


def _f64(t) -> np.ndarray:
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=F64)


def forward(X, W_hat, A, B, s: float, materialize: bool = True):
    """Y = X W_hat^T + s (U B^T), U = bf16(X A^T).  Returns (Y, U)."""
    X, W_hat, A, B = _f64(X), _f64(W_hat), _f64(A), _f64(B)
    U = X @ A.T
    if materialize:
        U = bf16(U)
    Y = X @ W_hat.T + F64(s) * (U @ B.T)
    return Y, U


def backward(X, W_hat, A, B, s: float, dY, U=None, materialize: bool = True):
    """Gradients of <dY, Y> for the forward above.

    V = bf16(dY B); dX = dY W_hat + s V A; dA = s V^T X; dB = s dY^T U.
    No gradient for W_hat: it is frozen ([P3] "Where the gradients actually go").
    """
    X, W_hat, A, B, dY = _f64(X), _f64(W_hat), _f64(A), _f64(B), _f64(dY)
    if U is None:
        U = X @ A.T
        if materialize:
            U = bf16(U)
    else:
        U = _f64(U)
    V = dY @ B
    if materialize:
        V = bf16(V)
    s = F64(s)
    dX = dY @ W_hat + s * (V @ A)
    dA = s * (V.T @ X)
    dB = s * (dY.T @ U)
    return dict(dX=dX, dA=dA, dB=dB, V=V, U=U)


def merge(W_hat, A, B, s: float) -> np.ndarray:
    """Adapter merge: W' = W_hat + s B A as a bf16 weight.

    [P2] FAQ "Does QLoRA introduce inference latency overhead once the model is
    fine-tuned and deployed?": the base is dequantized to 16 bits and the
    adapter folded in, W = W_dequant + (alpha / r) B A.  [P3] "Pitfalls" and
    "How it's used in practice" (merge_and_unload): the merge happens in 16
    bits; a quantized model is made by quantizing the merged weight again.

    The pages fix no summation order.  This reading, in fp32 with one rounding
    per step:
      d  = sum over j = 0 .. r-1, in that order, of B[n, j] A[j, k]
           (each product of two bf16 values is exact in fp32; each partial sum
           is rounded to fp32),
      t  = fl32(fl32(s) d),
      W' = bf16(fl32(W_hat + t)).
    The fp64 sums below are the fp32 additions themselves (formats.py: one
    IEEE operation on fp32 operands, rounded through float64).
    """
    W_hat, A, B = _f64(W_hat), _f64(A), _f64(B)
    d = np.zeros(W_hat.shape, dtype=F64)
    for j in range(A.shape[0]):
        d = fl32(d + np.outer(B[:, j], A[j, :]))
    t = fl32(fl32(s) * d)
    return bf16(fl32(W_hat + t))


def adapter_param_count(d: int, k: int, r: int) -> int:
    """[P3] "Prerequisite: LoRA's low-rank update": r (d + k) trainable numbers."""
    return r * (d + k)


# ----------------------------------------------------------- gated MLP chain
def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    return x * sigmoid(x)


def mlp_forward(X, Wg, Ag, Bg, Wu, Au, Bu, Wd, Ad, Bd, s: float, materialize: bool = True):
    """SiLU-gated MLP through three QLoRA linears.

    The pages only say that every linear layer gets an adapter ([P3] "Seeing it
    in code": gate_proj, up_proj, down_proj among the target modules).  The
    block itself is read as the usual gated MLP: g = Lg(X), u = Lu(X),
    h = silu(g) * u, y = Ld(h).  silu(x) = x * sigmoid(x).  g, u and h are
    materialized as bf16.
    """
    rb = bf16 if materialize else (lambda v: v)
    g, Ug = forward(X, Wg, Ag, Bg, s, materialize)
    u, Uu = forward(X, Wu, Au, Bu, s, materialize)
    g, u = rb(g), rb(u)
    h = rb(silu(g) * u)
    y, Ud = forward(h, Wd, Ad, Bd, s, materialize)
    return dict(y=y, g=g, u=u, h=h, Ug=Ug, Uu=Uu, Ud=Ud)


def mlp_backward(X, Wg, Ag, Bg, Wu, Au, Bu, Wd, Ad, Bd, s: float, dy, fwd: dict,
                 materialize: bool = True):
    """Backward of mlp_forward.

    dh = bf16(dX of Ld); dg = bf16(dh * u * sigmoid(g) * (1 + g (1 - sigmoid(g))));
    du = bf16(dh * silu(g)); dX = dX_g + dX_u.
    """
    rb = bf16 if materialize else (lambda v: v)
    g, u, h = fwd["g"], fwd["u"], fwd["h"]
    bd = backward(h, Wd, Ad, Bd, s, dy, U=fwd["Ud"], materialize=materialize)
    dh = rb(bd["dX"])
    sg = sigmoid(g)
    dg = rb(dh * u * sg * (1.0 + g * (1.0 - sg)))
    du = rb(dh * silu(g))
    bg = backward(X, Wg, Ag, Bg, s, dg, U=fwd["Ug"], materialize=materialize)
    bu = backward(X, Wu, Au, Bu, s, du, U=fwd["Uu"], materialize=materialize)
    return dict(dX=bg["dX"] + bu["dX"], dh=dh, dg=dg, du=du,
                dAg=bg["dA"], dBg=bg["dB"], dAu=bu["dA"], dBu=bu["dB"],
                dAd=bd["dA"], dBd=bd["dB"])
