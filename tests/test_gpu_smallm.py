"""GPU parity of the small-token forward (M <= 16 tokens: the split-K cluster
kernel) against the oracle, on shapes that exercise its tiling: ragged N,
K slices that are not whole code stages, a short last slice, several weight
tiles per cluster (double-buffered accumulators), no adapter and rank 64,
both constant forms and both output types."""
import numpy as np
import pytest
import torch

from oracle import lora
from tests._parity import np64, assert_fp_close, assert_bf16_within_ulp
from tests.test_gpu_linear import make_case, oracle_weight

pytestmark = pytest.mark.gpu

CASES = [
    # N, K, M, r, s
    (5120, 1408, 16, 16, 2.0),     # 22 K-blocks: 8 slices of 3 (last 1); 40 tiles, several per cluster
    (1000, 1344, 1, 64, 0.25),     # 21 K-blocks: 7 slices of 3; ragged N; one token; rank 64
    (2056, 4096, 7, 0, 1.0),       # no adapter; odd token count; N = 8 mod 16
    (384, 192, 4, 8, 0.5),         # 3 K-blocks: a 3-CTA cluster, one sub-step per slice
]


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


def run_fwd(q, W, X, A, B, r, s, dq, out_dtype):
    dev = "cuda"
    N, K = W.shape
    M = X.shape[0]
    w = q.quantize_weight(W.to(dev), dq=dq)
    Y = torch.empty(M, N, dtype=out_dtype, device=dev)
    U = torch.empty(M, r, dtype=torch.bfloat16, device=dev) if r else None
    ws = torch.empty(max(16, q.qlora_workspace_size(q.QL_OP_FWD, M, N, K, r)), dtype=torch.uint8, device=dev)
    q.qlora_linear_fwd(w, X.to(dev), A.to(dev) if r else None, B.to(dev) if r else None, r, s, Y, U_out=U, ws=ws)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    return Y, U


@pytest.mark.parametrize("N,K,M,r,s", CASES)
@pytest.mark.parametrize("dq", [True, False])
def test_small_token_forward(q, N, K, M, r, s, dq):
    W, X, A, B, _ = make_case(N, K, M, r, seed=40 + N + K + M + r)
    What = oracle_weight(W, dq)
    if r:
        ref, U_ref = lora.forward(X, What, A, B, s)
    else:
        ref = np64(X) @ What.T
    Y32, U = run_fwd(q, W, X, A, B, r, s, dq, torch.float32)
    assert_fp_close(np64(Y32), ref, f"Y fp32 N={N} K={K} M={M}")
    Ybf, _ = run_fwd(q, W, X, A, B, r, s, dq, torch.bfloat16)
    assert_bf16_within_ulp(Ybf, ref, f"Y bf16 N={N} K={K} M={M}", abs_rms=1e-3)
    if r:
        assert_bf16_within_ulp(U, U_ref, "U", abs_rms=1e-4)


def test_small_token_forward_is_deterministic(q):
    N, K, M, r, s = 5120, 1408, 16, 16, 2.0
    W, X, A, B, _ = make_case(N, K, M, r, seed=77)
    a, _ = run_fwd(q, W, X, A, B, r, s, True, torch.float32)
    b, _ = run_fwd(q, W, X, A, B, r, s, True, torch.float32)
    assert torch.equal(a, b)
