"""GPU parity of the QLoRA linear (qlora_linear_fwd / qlora_linear_bwd) against
the oracle: fp32 outputs within the stated tolerance of the float64 oracle,
bf16 outputs within one bf16 ulp, the saved U within one bf16 ulp."""
import numpy as np
import pytest
import torch

from oracle import lora, nf4
from synthetic import inputs as S
from tests._parity import np64, assert_fp_close, assert_bf16_within_ulp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


def oracle_weight(W_cpu, dq=True):
    packed, c, _ = nf4.quantize(W_cpu)
    if dq:
        e, s2, mu = nf4.double_quant(c)
        c = nf4.dq_constants(e, s2, mu)
    N, K = W_cpu.shape
    return nf4.dequant(packed, N * K, c, out="bf16").reshape(N, K)


def make_case(N, K, M, r, seed, wstd=0.02):
    W = S.custom_weight(N, K, wstd, seed)
    X = S.normal((M, K), 1.0, seed + 1, dtype=torch.bfloat16)
    A = S.uniform((r, K), 1.0 / np.sqrt(K), seed + 2) if r else None
    B = S.normal((N, r), 0.01, seed + 3, dtype=torch.bfloat16) if r else None
    dY = S.normal((M, N), 1.0, seed + 4, dtype=torch.bfloat16)
    return W, X, A, B, dY


def run_gpu(q, W, X, A, B, dY, r, s, dq=True, out_dtype=torch.float32, accumulate=False):
    dev = "cuda"
    N, K = W.shape
    M = X.shape[0]
    w = q.quantize_weight(W.to(dev), dq=dq)
    Xd, dYd = X.to(dev), dY.to(dev)
    Ad = A.to(dev) if r else None
    Bd = B.to(dev) if r else None
    Y = torch.empty(M, N, dtype=out_dtype, device=dev)
    U = torch.empty(M, max(r, 1), dtype=torch.bfloat16, device=dev) if r else None
    wsf = torch.empty(max(16, q.qlora_workspace_size(q.QL_OP_FWD, M, N, K, r)), dtype=torch.uint8, device=dev)
    q.qlora_linear_fwd(w, Xd, Ad, Bd, r, s, Y, U_out=U, ws=wsf)
    dX = torch.zeros(M, K, dtype=out_dtype, device=dev)
    if accumulate:
        dX.fill_(0.5)
    dA = torch.empty(max(r, 1), K, dtype=torch.float32, device=dev)
    dB = torch.empty(N, max(r, 1), dtype=torch.float32, device=dev)
    wsb = torch.empty(max(16, q.qlora_workspace_size(q.QL_OP_BWD, M, N, K, r)), dtype=torch.uint8, device=dev)
    q.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, r, s, U, dX, dA, dB, accumulate_dx=accumulate, ws=wsb)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    return dict(Y=Y, U=U, dX=dX, dA=dA, dB=dB)


def run_oracle(W, X, A, B, dY, r, s, dq=True):
    What = oracle_weight(W, dq)
    if r == 0:
        Y = np64(X) @ What.T
        return dict(Y=Y, U=None, dX=np64(dY) @ What, dA=None, dB=None)
    Y, U = lora.forward(X, What, A, B, s)
    g = lora.backward(X, What, A, B, s, dY, U=U)
    return dict(Y=Y, **g)


SHAPES = [
    # N, K, M, r, s
    (256, 512, 16, 8, 2.0),          # the small single-linear workload
    (320, 448, 200, 16, 2.0),        # N not a multiple of 256, K of 256, M of 128
    (136, 192, 1, 64, 0.25),         # one token, r = 64
    (512, 1024, 130, 16, 0.75),      # s not a power of two
    (256, 256, 64, 0, 1.0),          # no adapter
    (264, 192, 40, 16, 0.5),         # N = 8 mod 16: a half chunk at the end of each output row
    (384, 320, 600, 8, 1.0),         # two token tiles of 512, ragged N and M, stage ring wraps
]


@pytest.mark.parametrize("N,K,M,r,s", SHAPES)
@pytest.mark.parametrize("dq", [True, False])
def test_fwd_bwd_fp32_outputs(q, N, K, M, r, s, dq):
    case = make_case(N, K, M, r, seed=7 + N + K + M + r)
    got = run_gpu(q, *case, r, s, dq=dq)
    ref = run_oracle(*case, r, s, dq=dq)
    assert_fp_close(np64(got["Y"]), ref["Y"], "Y")
    assert_fp_close(np64(got["dX"]), ref["dX"], "dX")
    if r:
        assert_bf16_within_ulp(got["U"][:, :r], ref["U"], "U", abs_rms=1e-4)
        assert_fp_close(np64(got["dA"][:r]), ref["dA"], "dA")
        assert_fp_close(np64(got["dB"][:, :r]), ref["dB"], "dB")


@pytest.mark.parametrize("N,K,M,r,s", SHAPES)
def test_bf16_outputs_within_one_ulp(q, N, K, M, r, s):
    case = make_case(N, K, M, r, seed=11 + N + K + M + r)
    got = run_gpu(q, *case, r, s, out_dtype=torch.bfloat16)
    ref = run_oracle(*case, r, s)
    # The adapter term enters the accumulator as U bf16(s B)^T: exact when s is a
    # power of two; otherwise bf16(s B) carries one rounding (relative 2^-9), a
    # bound of about 1e-4 * rms(Y) here, so near-zero outputs get 1e-3 * rms.
    abs_y = 0.0 if float(np.log2(s)).is_integer() else 1e-3
    assert_bf16_within_ulp(got["Y"], ref["Y"], "Y bf16", abs_rms=abs_y)
    assert_bf16_within_ulp(got["dX"], ref["dX"], "dX bf16", abs_rms=1e-3)


def test_accumulate_dx(q):
    N, K, M, r, s = 256, 512, 40, 16, 2.0
    case = make_case(N, K, M, r, seed=3)
    got = run_gpu(q, *case, r, s, accumulate=True)
    ref = run_oracle(*case, r, s)
    assert_fp_close(np64(got["dX"]) - 0.5, ref["dX"], "dX accumulate")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_projection_workload_full(q, out_dtype):
    """The 4096 x 4096 projection with 4096 tokens, r = 16, alpha = 32, at full size
    (bf16 Y and dX are what the timed step writes)."""
    w = S.WORKLOADS["c2"]
    d = S.linear_inputs(w, 0)
    got = run_gpu(q, d["W"], d["X"], d["A"], d["B"], d["dY"], w.r, w.s, out_dtype=out_dtype)
    ref = run_oracle(d["W"], d["X"], d["A"], d["B"], d["dY"], w.r, w.s)
    for k in ("Y", "dX"):
        if out_dtype == torch.bfloat16:
            assert_bf16_within_ulp(got[k], ref[k], k + " bf16", abs_rms=1e-3)
        else:
            assert_fp_close(np64(got[k]), ref[k], k)
    assert_fp_close(np64(got["dA"]), ref["dA"], "dA")
    assert_fp_close(np64(got["dB"]), ref["dB"], "dB")
    assert_bf16_within_ulp(got["U"], ref["U"], "U", abs_rms=1e-4)
