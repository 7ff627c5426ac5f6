"""The large workloads at full size: the 70B-shaped layer linears and the
small-token 28672 x 8192 weight.  Outputs are checked against the oracle on
sampled entries it can compute one by one (sampled weight rows and token
rows), and full-tensor properties that hold at any size:
  <dY, Y> = <dX, X>   (the backward is the adjoint of the forward)
  <dA, A> = <dB, B>   (both equal s <U, V>)
"""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import lora, nf4
from synthetic import inputs as S
from tests._parity import np64, assert_fp_close, assert_bf16_within_ulp, adjoint_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


def oracle_rows(W_dev, rows):
    """Oracle dequantized rows of a (double-quantized) weight: the mean needs
    every block constant, the codes only the sampled rows."""
    N, K = W_dev.shape
    kb = K // 64
    c = np.empty(N * kb, dtype=np.float64)
    step = max(1, (1 << 26) // K)
    for r0 in range(0, N, step):
        part = W_dev[r0:r0 + step].cpu()
        cc, finite = nf4.block_absmax(part)
        assert finite
        c[r0 * kb:(r0 + part.shape[0]) * kb] = cc
    e, s2, mu = nf4.double_quant(c)
    chat = nf4.dq_constants(e, s2, mu)
    out = []
    for n in rows:
        wr = W_dev[int(n)].cpu()
        packed, _, _ = nf4.quantize(wr)
        out.append(nf4.dequant(packed, K, chat[int(n) * kb:(int(n) + 1) * kb]))
    return np.stack(out)


def run_linear(q, W, X, A, B, dY, r, s, out_dtype=torch.float32, bwd=True):
    dev = W.device
    M, K = X.shape
    N = W.shape[0]
    w = q.quantize_weight(W)
    Y = torch.empty(M, N, dtype=out_dtype, device=dev)
    U = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(16, q.qlora_workspace_size(q.QL_OP_FWD, M, N, K, r),
                         q.qlora_workspace_size(q.QL_OP_BWD, M, N, K, r)), dtype=torch.uint8, device=dev)
    q.qlora_linear_fwd(w, X, A, B, r, s, Y, U_out=U, ws=ws)
    res = dict(Y=Y, U=U)
    if bwd:
        dX = torch.empty(M, K, dtype=torch.float32, device=dev)
        dA = torch.empty(r, K, dtype=torch.float32, device=dev)
        dB = torch.empty(N, r, dtype=torch.float32, device=dev)
        q.qlora_linear_bwd(w, X, dY, A, B, r, s, U, dX, dA, dB, ws=ws)
        res.update(dX=dX, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    return res


def sampled_y_check(Y, X, Wrows, rows, U, Bm, s, what, bf16_out=False):
    ref = np64(X) @ Wrows.T + s * (np64(U) @ np64(Bm[rows]).T)
    got = Y[:, rows]
    if bf16_out:
        assert_bf16_within_ulp(got, ref, what, abs_rms=1e-3)
    else:
        assert_fp_close(np64(got), ref, what)


@pytest.mark.parametrize("j", [0, 1, 4, 6])          # q, k (GQA 1024 rows), gate, down
def test_layer_linears_full_size(q, j):
    w = S.WORKLOADS["c4"]
    lin = w.linears[j]
    d = S.linear_inputs(w, j, device="cuda")
    res = run_linear(q, d["W"], d["X"], d["A"], d["B"], d["dY"], w.r, w.s)
    rng = np.random.default_rng(j)
    rows = np.unique(np.concatenate([rng.integers(0, lin.N, 12), [0, lin.N - 1]]))
    Wr = oracle_rows(d["W"], rows)
    # U from the oracle's own bf16(X A^T) for the sampled entries
    U_ref = F.bf16(np64(d["X"]) @ np64(d["A"]).T)
    assert_bf16_within_ulp(res["U"], U_ref, "U", abs_rms=1e-4)
    sampled_y_check(res["Y"], d["X"], Wr, rows, U_ref, d["B"], w.s, f"Y[{lin.name}] sampled rows")
    V_ref = np64(d["dY"]) @ np64(d["B"])
    dY, Y, dX, X = np64(d["dY"]), np64(res["Y"]), np64(res["dX"]), np64(d["X"])
    lhs, rhs = float((dY * Y).sum()), float((dX * X).sum())
    assert abs(lhs - rhs) <= adjoint_bound(w.s, U_ref, V_ref, (dY, Y), (dX, X)), (lhs, rhs)
    dA, A, dB, B = np64(res["dA"]), np64(d["A"]), np64(res["dB"]), np64(d["B"])
    lhs, rhs = float((dA * A).sum()), float((dB * B).sum())
    assert abs(lhs - rhs) <= adjoint_bound(w.s, U_ref, V_ref, (dA, A), (dB, B)), (lhs, rhs)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_small_token_forward_full_size(q, M):
    w = S.WORKLOADS["c5"]
    lin = w.linears[0]
    d = S.linear_inputs(w, 0, M=M, device="cuda")
    for out_dtype in (torch.float32, torch.bfloat16):
        res = run_linear(q, d["W"], d["X"], d["A"], d["B"], d["dY"], w.r, w.s, out_dtype=out_dtype, bwd=False)
        if out_dtype == torch.float32:
            Y32 = res["Y"]
        else:
            Ybf = res["Y"]
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([rng.integers(0, lin.N, 24), [0, 127, 128, lin.N - 1]]))
    Wr = oracle_rows(d["W"], rows)
    U_ref = F.bf16(np64(d["X"]) @ np64(d["A"]).T)
    sampled_y_check(Y32, d["X"], Wr, rows, U_ref, d["B"], w.s, f"Y M={M}")
    sampled_y_check(Ybf, d["X"], Wr, rows, U_ref, d["B"], w.s, f"Y bf16 M={M}", bf16_out=True)
