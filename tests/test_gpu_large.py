"""The large workloads at full size: the 70B-shaped layer linears and the
small-token 28672 x 8192 weight, against the oracle.
  - dA [r, K] and dB [N, r] element by element in full (small products over
    the 2048 tokens);
  - Y on sampled output columns (sampled weight rows, every token);
  - dX on sampled 64-column blocks (the weight's block columns, every token)
    and, where the whole weight dequantizes in seconds on the host (k and v,
    1024 x 8192), on sampled token rows;
  - full-tensor properties that hold at any size:
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


def oracle_constants(W_dev):
    """Oracle reconstructed block constants of a (double-quantized) weight: the
    mean needs every block constant, so all of them are computed (in row
    chunks copied from the device)."""
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
    return nf4.dq_constants(e, s2, mu)


def oracle_col_blocks(W_dev, kbs, chat=None):
    """Oracle dequantized weight columns [64 kb, 64 kb + 64) for each kb in
    kbs, every row: each row's slice is exactly one 64-block, so only those
    blocks are quantized."""
    N, K = W_dev.shape
    nkb = K // 64
    chat = oracle_constants(W_dev) if chat is None else chat
    cols = []
    for kb in kbs:
        blk = W_dev[:, 64 * kb:64 * kb + 64].cpu().contiguous()
        packed, _, _ = nf4.quantize(blk)
        cols.append(nf4.dequant(packed, N * 64, chat[np.arange(N) * nkb + kb]).reshape(N, 64))
    return np.concatenate(cols, axis=1)


def oracle_full(W_dev, chat=None):
    """The whole oracle dequantized weight (for small weights only)."""
    N, K = W_dev.shape
    chat = oracle_constants(W_dev) if chat is None else chat
    packed, _, _ = nf4.quantize(W_dev.cpu())
    return nf4.dequant(packed, N * K, chat).reshape(N, K)


def oracle_rows(W_dev, rows, chat=None):
    """Oracle dequantized rows of a (double-quantized) weight."""
    N, K = W_dev.shape
    kb = K // 64
    chat = oracle_constants(W_dev) if chat is None else chat
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


@pytest.mark.parametrize("j", range(7))     # q, k, v (GQA, 1024 rows), o, gate, up, down
def test_layer_linears_full_size(q, j):
    w = S.WORKLOADS["c4"]
    lin = w.linears[j]
    d = S.linear_inputs(w, j, device="cuda")
    res = run_linear(q, d["W"], d["X"], d["A"], d["B"], d["dY"], w.r, w.s)
    chat = oracle_constants(d["W"])
    rng = np.random.default_rng(j)
    rows = np.unique(np.concatenate([rng.integers(0, lin.N, 12), [0, lin.N - 1]]))
    Wr = oracle_rows(d["W"], rows, chat)
    # U from the oracle's own bf16(X A^T) for the sampled entries
    X64, A64, B64, dY64 = np64(d["X"]), np64(d["A"]), np64(d["B"]), np64(d["dY"])
    U_ref = F.bf16(X64 @ A64.T)
    assert_bf16_within_ulp(res["U"], U_ref, "U", abs_rms=1e-4)
    sampled_y_check(res["Y"], d["X"], Wr, rows, U_ref, d["B"], w.s, f"Y[{lin.name}] sampled rows")
    # adapter gradients in full and dX on sampled block columns, from the
    # oracle's backward (its own bf16 V = bf16(dY B))
    kbs = np.unique(np.concatenate([rng.integers(0, lin.K // 64, 2), [0, lin.K // 64 - 1]]))
    Wc = oracle_col_blocks(d["W"], kbs, chat)
    cols = np.concatenate([np.arange(64 * kb, 64 * kb + 64) for kb in kbs])
    g = lora.backward(X64[:, cols], Wc, A64[:, cols], B64, w.s, dY64, U=U_ref)
    assert_fp_close(np64(res["dX"])[:, cols], g["dX"], f"dX[{lin.name}] sampled block columns")
    assert_fp_close(np64(res["dB"]), g["dB"], f"dB[{lin.name}]")
    dA_ref = w.s * (g["V"].T @ X64)
    assert_fp_close(np64(res["dA"]), dA_ref, f"dA[{lin.name}]")
    if lin.N * lin.K <= (1 << 23):
        # the whole weight is small enough: dX on sampled token rows too
        Wf = oracle_full(d["W"], chat)
        trows = np.unique(np.concatenate([rng.integers(0, w.M, 14), [0, w.M - 1]]))
        gr = lora.backward(X64[trows], Wf, A64, B64, w.s, dY64[trows], U=U_ref[trows])
        assert_fp_close(np64(res["dX"])[trows], gr["dX"], f"dX[{lin.name}] sampled token rows")
    V_ref = dY64 @ B64
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
