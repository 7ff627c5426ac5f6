"""AdamW update of the adapter parameters (oracle; tests only).

TEST INFRASTRUCTURE ONLY (see the package docstring).  float64 numpy.

Sources:
  [P1] "Lesson 4 of the Finetuning Sessions", "Inside QLoRA: NF4 and Paged
       Optimizers" (optimizer states in NVIDIA Unified Memory, offloaded to CPU
       RAM when the GPU is full and brought back for the next update);
  [P2] "QLoRA: Quantize Base Weights to 4-Bit", §2.3 (AdamW states registered
       in unified memory, paged out during activation spikes);
  [P3] "QLoRA — Fine-Tuning a 65B Model on One GPU", "Paged optimizers:
       surviving the spikes" (paging changes where the states live, not the
       update); "How it's used in practice" (optim="paged_adamw_32bit").
The pages give no update formula: paging moves the states, the arithmetic is
AdamW with decoupled weight decay.  Only A and B are updated ([P3] "Where the
gradients actually go").

Reading (the usual AdamW, decoupled weight decay applied to the parameter
before the moment step), for step t = 1, 2, ...:
    p <- p (1 - lr wd)
    m <- b1 m + (1 - b1) g
    v <- b2 v + (1 - b2) g^2
    p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
States m, v and parameters are fp32 in "paged_adamw_32bit"; this oracle keeps
float64 and leaves the fp32 rounding to the caller's tolerance.

Parity: pinned by tests/test_oracle_adamw.py (the first step moves every
parameter by lr sign(g) when eps is negligible, weight decay alone scales p,
zero gradients keep p up to decay, and torch.optim.AdamW agrees on random
cases).
"""
from __future__ import annotations

import numpy as np

from .formats import F64


def adamw_step(p, g, m, v, t: int, lr: float, b1: float = 0.9, b2: float = 0.999, eps: float = 1e-8,
               wd: float = 0.0):
    """One AdamW step; returns (p, m, v) as new float64 arrays."""
    p, g, m, v = (np.asarray(a, dtype=F64) for a in (p, g, m, v))
    p = p * (1.0 - lr * wd)
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    mhat = m / (1.0 - b1 ** t)
    vhat = v / (1.0 - b2 ** t)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v


def adamw_step_fp32(p, g, m, v, t: int, lr: float, b1: float = 0.9, b2: float = 0.999, eps: float = 1e-8,
                    wd: float = 0.0):
    """The same step as single fp32 operations in a fixed order (what a kernel
    with fp32 states computes; "paged_adamw_32bit").  Constants are fp32, the
    bias corrections from the fp32 betas (so 1 - b1 and the t = 1 correction
    are the same number):
        b1, b2, lr, eps, wd = fl32(.);  keep = fl32(1 - lr wd)  (product in float64)
        c1 = fl32(1 - b1^t), c2 = fl32(1 - b2^t)   (power in float64)
        p  = fl32(p keep)
        m  = fl32(fl32(b1 m) + fl32((1 - b1) g))
        v  = fl32(fl32(b2 v) + fl32(fl32((1 - b2) g) g))
        d  = fl32(fl32(sqrt(fl32(v / c2))) + eps)
        p  = fl32(p - fl32(lr fl32(fl32(m / c1) / d)))
    Each line's float64 operation followed by fl32 is the fp32 operation itself
    (formats.py; the same holds for sqrt).  Returns (p, m, v) as fp32 values."""
    from .formats import fl32
    f = lambda x: fl32(np.asarray(x, dtype=F64))
    p, g, m, v = f(p), f(g), f(m), f(v)
    lr_, b1_, b2_, eps_ = (float(f(x)) for x in (lr, b1, b2, eps))
    keep = float(f(1.0 - lr_ * float(f(wd))))   # from the fp32 lr and wd, product in float64
    c1, c2 = float(f(1.0 - b1_ ** t)), float(f(1.0 - b2_ ** t))
    omb1, omb2 = float(f(1.0 - b1_)), float(f(1.0 - b2_))
    p = f(p * keep)
    m = f(f(b1_ * m) + f(omb1 * g))
    v = f(f(b2_ * v) + f(f(omb2 * g) * g))
    d = f(f(np.sqrt(f(v / c2))) + eps_)
    p = f(p - f(lr_ * f(f(m / c1) / d)))
    return p, m, v
