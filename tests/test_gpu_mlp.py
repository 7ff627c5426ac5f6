"""GPU parity of the SiLU-gated MLP chain (three QLoRA linears + the gate glue)
against the oracle, and of the gate kernels element by element."""
import numpy as np
import pytest
import torch

from oracle import lora, nf4
from synthetic import inputs as S
from tests._parity import np64, assert_fp_close, assert_bf16_within_ulp, adjoint_bound, assert_chain_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


def test_silu_gate_kernels(q):
    n = 8 * 40000
    g = S.normal((n,), 2.0, 1, dtype=torch.bfloat16)
    u = S.normal((n,), 1.0, 2, dtype=torch.bfloat16)
    dh = S.normal((n,), 1.0, 3, dtype=torch.bfloat16)
    g[:8] = torch.tensor([0.0, -0.0, 30.0, -30.0, 88.0, -88.0, 1e-3, -1e-3], dtype=torch.bfloat16)
    gd, ud, dhd = g.cuda(), u.cuda(), dh.cuda()
    h = torch.empty_like(gd)
    dg, du = torch.empty_like(gd), torch.empty_like(gd)
    q.qlora_silu_gate_fwd(gd, ud, h)
    q.qlora_silu_gate_bwd(dhd, gd, ud, dg, du)
    torch.cuda.synchronize()
    G, Uu, DH = np64(g), np64(u), np64(dh)
    sg = lora.sigmoid(G)
    assert_bf16_within_ulp(h, lora.silu(G) * Uu, "h")
    assert_bf16_within_ulp(dg, DH * Uu * sg * (1 + G * (1 - sg)), "dg")
    assert_bf16_within_ulp(du, DH * lora.silu(G), "du")


def _oracle_weight(W):
    packed, c, _ = nf4.quantize(W)
    e, s2, mu = nf4.double_quant(c)
    N, K = W.shape
    return nf4.dequant(packed, N * K, nf4.dq_constants(e, s2, mu)).reshape(N, K)


def chain_bounds(c, f, b, Wg, Wu, Wd, s):
    """Largest move of y and dX if every bf16 intermediate (h, U of the down
    linear; dg, du, V of the gate/up linears) were one ulp off."""
    e = 2.0 ** -7
    ab = np.abs
    yb = e * (ab(f["h"]) @ ab(Wd).T + s * ab(f["Ud"]) @ ab(np64(c["Bd"])).T)
    Vg, Vu = b["dg"] @ np64(c["Bg"]), b["du"] @ np64(c["Bu"])
    dxb = e * (ab(b["dg"]) @ ab(Wg) + ab(b["du"]) @ ab(Wu)
               + s * (ab(Vg) @ ab(np64(c["Ag"])) + ab(Vu) @ ab(np64(c["Au"]))))
    return yb, dxb


def _mlp_case(D, H, M, r, seed):
    Wg = S.custom_weight(H, D, 0.02, seed)
    Wu = S.custom_weight(H, D, 0.02, seed + 1)
    Wd = S.custom_weight(D, H, 0.02, seed + 2)
    Ag = S.uniform((r, D), 1 / np.sqrt(D), seed + 3)
    Au = S.uniform((r, D), 1 / np.sqrt(D), seed + 4)
    Ad = S.uniform((r, H), 1 / np.sqrt(H), seed + 5)
    Bg = S.normal((H, r), 0.01, seed + 6, dtype=torch.bfloat16)
    Bu = S.normal((H, r), 0.01, seed + 7, dtype=torch.bfloat16)
    Bd = S.normal((D, r), 0.01, seed + 8, dtype=torch.bfloat16)
    X = S.normal((M, D), 1.0, seed + 9, dtype=torch.bfloat16)
    dy = S.normal((M, D), 1.0, seed + 10, dtype=torch.bfloat16)
    return dict(Wg=Wg, Wu=Wu, Wd=Wd, Ag=Ag, Au=Au, Ad=Ad, Bg=Bg, Bu=Bu, Bd=Bd, X=X, dy=dy)


def _run_gpu_mlp(q, c, r, s):
    from bit_nf4_quantized_10_b200.mlp import QLoRAMLP
    dev = "cuda"
    wg, wu, wd = (q.quantize_weight(c[k].to(dev)) for k in ("Wg", "Wu", "Wd"))
    t = {k: c[k].to(dev) for k in ("Ag", "Au", "Ad", "Bg", "Bu", "Bd", "X", "dy")}
    M = c["X"].shape[0]
    mlp = QLoRAMLP(wg, wu, wd, t["Ag"], t["Bg"], t["Au"], t["Bu"], t["Ad"], t["Bd"], r, s, M)
    y = torch.empty(M, c["Wd"].shape[0], dtype=torch.bfloat16, device=dev)
    mlp.forward(t["X"], y)
    mlp.backward(t["X"], t["dy"])
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    return mlp, y


def test_mlp_chain_reduced_tokens(q):
    """A reduced gated MLP (1024 -> 2816 -> 1024), r = 64, alpha = 16, 256
    tokens: every output and every gradient against the oracle."""
    D, H, M, r, s = 1024, 2816, 256, 64, 0.25
    c = _mlp_case(D, H, M, r, seed=300)
    mlp, y = _run_gpu_mlp(q, c, r, s)
    Wg, Wu, Wd = _oracle_weight(c["Wg"]), _oracle_weight(c["Wu"]), _oracle_weight(c["Wd"])
    args = (c["X"], Wg, c["Ag"], c["Bg"], Wu, c["Au"], c["Bu"], Wd, c["Ad"], c["Bd"], s)
    f = lora.mlp_forward(*args)
    b = lora.mlp_backward(*args, c["dy"], f)
    yb, dxb = chain_bounds(c, f, b, Wg, Wu, Wd, s)
    assert_chain_close(np64(y), f["y"], yb, "y")
    assert_chain_close(np64(mlp.dX), b["dX"], dxb, "dX")
    for name, got in (("dAg", mlp.dAg), ("dBg", mlp.dBg), ("dAu", mlp.dAu), ("dBu", mlp.dBu),
                      ("dAd", mlp.dAd), ("dBd", mlp.dBd)):
        assert_chain_close(np64(got), b[name], np.inf, name)


def _rows_of(d, rows, keys):
    return {k: (v[rows] if k in keys else v) for k, v in d.items()}


def test_mlp_chain_full_size(q):
    """The 7B MLP workload at full size (8192 tokens, r = 64).  The oracle runs
    the whole chain on every token; the six adapter gradients are compared
    element by element in full, and y and dX (per token) on sampled token rows
    with the bound of a one-ulp flip in every bf16 intermediate."""
    w = S.WORKLOADS["c3"]
    D, H, M, r, s = 4096, 11008, w.M, w.r, w.s
    c = _mlp_case(D, H, M, r, seed=3000)
    mlp, y = _run_gpu_mlp(q, c, r, s)
    Wg, Wu, Wd = _oracle_weight(c["Wg"]), _oracle_weight(c["Wu"]), _oracle_weight(c["Wd"])
    args = (c["X"], Wg, c["Ag"], c["Bg"], Wu, c["Au"], c["Bu"], Wd, c["Ad"], c["Bd"], s)
    f = lora.mlp_forward(*args)
    b = lora.mlp_backward(*args, c["dy"], f)
    for name, got in (("dAg", mlp.dAg), ("dBg", mlp.dBg), ("dAu", mlp.dAu), ("dBu", mlp.dBu),
                      ("dAd", mlp.dAd), ("dBd", mlp.dBd)):
        assert_fp_close(np64(got), b[name], name)
    rows = np.array([0, 1, 77, 1000, 4095, 4096, 6000, M - 1])
    sub = dict(c)
    sub["X"], sub["dy"] = c["X"][rows], c["dy"][rows]
    fr = _rows_of(f, rows, ("y", "g", "u", "h", "Ug", "Uu", "Ud"))
    br = _rows_of(b, rows, ("dX", "dh", "dg", "du"))
    yb, dxb = chain_bounds(sub, fr, br, Wg, Wu, Wd, s)
    assert_chain_close(np64(y[rows]), fr["y"], yb, "y rows")
    assert_chain_close(np64(mlp.dX[rows]), br["dX"], dxb, "dX rows")
