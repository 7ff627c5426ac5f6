"""GPU parity of the small-token forward (M <= 16 tokens) against the oracle,
on shapes that exercise its tiling: ragged N (a partial last 16-row block),
K ranges that end inside a warp's chunk, several K parts (one part is 4096
reduction elements for up to 8 tokens, 2048 above), token counts on both sides
of the 8-token tile, no adapter and rank 64, both constant forms and both
output types."""
import numpy as np
import pytest
import torch

from oracle import lora
from tests._parity import np64, assert_fp_close, assert_bf16_within_ulp
from tests.test_gpu_linear import make_case, oracle_weight

pytestmark = pytest.mark.gpu

CASES = [
    # N, K, M, r, s
    (5120, 1408, 16, 16, 2.0),     # two token tiles; 11 warp chunks of 128 in one part, 5 warps idle
    (1000, 1344, 1, 64, 0.25),     # one token; a last chunk of one block; N = 8 mod 16; rank 64
    (2056, 4096, 7, 0, 1.0),       # no adapter; odd token count; exactly one part
    (384, 192, 4, 8, 0.5),         # one warp chunk of 3 blocks; rank 8 (half an adapter tile)
    (1024, 9216, 9, 16, 2.0),      # 9 tokens (two tiles, one nearly empty); 5 parts, the last one half
    (264, 8256, 8, 32, 1.0),       # 8 tokens (one tile); 3 parts, the last one a single block
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
