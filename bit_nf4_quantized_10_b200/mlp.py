"""SiLU-gated MLP through three QLoRA linears (gate, up, down), forward and backward.

Host-side sequencing of C-ABI calls only; every step runs in the library's
kernels.  The pages adapt every linear layer of the block ("QLoRA — Fine-Tuning
a 65B Model on One GPU", "Seeing it in code": gate_proj, up_proj, down_proj);
the block is the usual gated MLP  y = Ld(silu(Lg(x)) * Lu(x)).
g, u and h are materialized as bf16; dX of the gate and up linears are summed
in fp32 (accumulate_dx), and dX is returned in fp32.
"""
from __future__ import annotations

import torch

from . import _lib as q


class QLoRAMLP:
    def __init__(self, wg, wu, wd, Ag, Bg, Au, Bu, Ad, Bd, r: int, s: float, M: int):
        self.wg, self.wu, self.wd = wg, wu, wd
        self.Ag, self.Bg, self.Au, self.Bu, self.Ad, self.Bd = Ag, Bg, Au, Bu, Ad, Bd
        self.r, self.s, self.M = r, s, M
        dev = Ag.device
        H, D = wg.rows, wg.cols
        bf = torch.bfloat16
        self.g = torch.empty(M, H, dtype=bf, device=dev)
        self.u = torch.empty(M, H, dtype=bf, device=dev)
        self.h = torch.empty(M, H, dtype=bf, device=dev)
        self.Ug = torch.empty(M, r, dtype=bf, device=dev)
        self.Uu = torch.empty(M, r, dtype=bf, device=dev)
        self.Ud = torch.empty(M, r, dtype=bf, device=dev)
        self.dh = torch.empty(M, H, dtype=bf, device=dev)
        self.dg = torch.empty(M, H, dtype=bf, device=dev)
        self.du = torch.empty(M, H, dtype=bf, device=dev)
        self.dX = torch.empty(M, D, dtype=torch.float32, device=dev)
        f32 = torch.float32
        self.dAg = torch.empty(r, D, dtype=f32, device=dev)
        self.dBg = torch.empty(H, r, dtype=f32, device=dev)
        self.dAu = torch.empty(r, D, dtype=f32, device=dev)
        self.dBu = torch.empty(H, r, dtype=f32, device=dev)
        self.dAd = torch.empty(r, H, dtype=f32, device=dev)
        self.dBd = torch.empty(D, r, dtype=f32, device=dev)
        ws = 0
        for w, K in ((wg, D), (wu, D), (wd, H)):
            ws = max(ws, q.qlora_workspace_size(q.QL_OP_FWD, M, w.rows, K, r),
                     q.qlora_workspace_size(q.QL_OP_BWD, M, w.rows, K, r))
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)

    def forward(self, X, y):
        r, s, ws = self.r, self.s, self.ws
        q.qlora_linear_fwd(self.wg, X, self.Ag, self.Bg, r, s, self.g, U_out=self.Ug, ws=ws)
        q.qlora_linear_fwd(self.wu, X, self.Au, self.Bu, r, s, self.u, U_out=self.Uu, ws=ws)
        q.qlora_silu_gate_fwd(self.g, self.u, self.h)
        q.qlora_linear_fwd(self.wd, self.h, self.Ad, self.Bd, r, s, y, U_out=self.Ud, ws=ws)

    def backward(self, X, dy):
        r, s, ws = self.r, self.s, self.ws
        q.qlora_linear_bwd(self.wd, self.h, dy, self.Ad, self.Bd, r, s, self.Ud, self.dh, self.dAd, self.dBd, ws=ws)
        q.qlora_silu_gate_bwd(self.dh, self.g, self.u, self.dg, self.du)
        q.qlora_linear_bwd(self.wg, X, self.dg, self.Ag, self.Bg, r, s, self.Ug, self.dX, self.dAg, self.dBg, ws=ws)
        q.qlora_linear_bwd(self.wu, X, self.du, self.Au, self.Bu, r, s, self.Uu, self.dX, self.dAu, self.dBu,
                           accumulate_dx=True, ws=ws)

    def flops(self) -> float:
        M, r = self.M, self.r
        tot = 0.0
        for w in (self.wg, self.wu, self.wd):
            N, K = w.rows, w.cols
            tot += 4.0 * M * N * K + 6.0 * M * r * (K + N)
        return tot
