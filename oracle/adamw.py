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
