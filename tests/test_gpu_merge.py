"""GPU parity of the adapter merge (qlora_merge) against the oracle.

The merged bf16 weight W' = W_hat + s B A is compared bit for bit with
oracle.lora.merge (both follow the same fp32 order), and the re-quantized
weight (codes and fp32 constants) bit for bit with the oracle's quantization of
that merged weight."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import lora, nf4
from synthetic import inputs as S
from tests._parity import bf16_bits_t, f32_bits_t, np_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


def make_case(N, K, r, s, dq, seed):
    W = S.custom_weight(N, K, 0.02, seed)
    A = S.uniform((r, K), 1.0 / np.sqrt(K), seed + 2)
    B = S.normal((N, r), 0.01, seed + 3, dtype=torch.bfloat16)
    packed, c, _ = nf4.quantize(W)
    if dq:
        e, s2, mu = nf4.double_quant(c)
        c = nf4.dq_constants(e, s2, mu)
    W_hat = nf4.dequant(packed, N * K, c, out="bf16").reshape(N, K)
    merged = lora.merge(W_hat, A.double().numpy(), B.double().numpy(), s)
    packed2, c2, _ = nf4.quantize(merged.reshape(-1))
    return W, A, B, W_hat, merged, packed2, c2


def run_merge(q, W, A, B, r, s, dq, want_w=True, want_codes=True):
    dev = "cuda"
    N, K = W.shape
    w = q.quantize_weight(W.to(dev), dq=dq)
    W_out = torch.empty(N, K, dtype=torch.bfloat16, device=dev) if want_w else None
    codes = torch.empty(N * K // 2, dtype=torch.uint8, device=dev) if want_codes else None
    absmax = torch.empty(N * K // 64, dtype=torch.float32, device=dev) if want_codes else None
    q.qlora_merge(w, A.to(dev) if r else None, B.to(dev) if r else None, r, s, W_out=W_out, codes_out=codes,
                  absmax_out=absmax)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    return w, W_out, codes, absmax


SHAPES = [
    # N, K, r, s
    (256, 512, 16, 2.0),      # the small single-linear shape
    (200, 320, 8, 0.75),      # N not a multiple of 8, K of 128; s not a power of two
    (72, 64, 1, 0.25),        # one 64-block per row, rank 1
    (136, 192, 64, 0.5),      # the largest rank
    (96, 128, 3, 1.0),        # a rank that is no multiple of 8
    (64, 128, 0, 2.0),        # no adapter: the merge is the dequantized weight
    # K = 16384 leaves 4 CTAs per 256-column tile, so each walks several 64-row
    # tiles (the next tile's B and codes load during the current one's sums)
    (520, 16384, 32, 0.75),   # ranks 17..32, a ragged last row tile of 8 rows
    (640, 16384, 64, 0.5),    # ranks 33..64
]


@pytest.mark.parametrize("N,K,r,s", SHAPES)
@pytest.mark.parametrize("dq", [True, False])
def test_merge_and_requantize_bit_exact(q, N, K, r, s, dq):
    W, A, B, W_hat, merged, packed2, c2 = make_case(N, K, r, s, dq, seed=41 + N + K + r)
    _, W_out, codes, absmax = run_merge(q, W, A, B, r, s, dq)
    assert np.array_equal(bf16_bits_t(W_out).reshape(-1), F.bf16_bits(merged).reshape(-1))
    assert np.array_equal(np_u8(codes), packed2)
    assert np.array_equal(f32_bits_t(absmax), F.f32_bits(c2))


def test_merge_outputs_alone_agree(q):
    N, K, r, s = 128, 256, 16, 2.0
    W, A, B, W_hat, merged, packed2, c2 = make_case(N, K, r, s, True, seed=5)
    _, W_only, _, _ = run_merge(q, W, A, B, r, s, True, want_codes=False)
    _, _, codes_only, absmax_only = run_merge(q, W, A, B, r, s, True, want_w=False)
    assert np.array_equal(bf16_bits_t(W_only).reshape(-1), F.bf16_bits(merged).reshape(-1))
    assert np.array_equal(np_u8(codes_only), packed2)
    assert np.array_equal(f32_bits_t(absmax_only), F.f32_bits(c2))


def test_zero_adapter_requantizes_to_the_original_codes(q):
    N, K, r = 64, 512, 16
    W, A, B, *_ = make_case(N, K, r, 2.0, True, seed=9)
    w, W_out, codes, _ = run_merge(q, W, A, B, r, 0.0, True)
    assert torch.equal(codes, w.codes)
    deq = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    q.nf4_dequant(w, deq)
    torch.cuda.synchronize()
    assert torch.equal(W_out.view(torch.int16), deq.view(torch.int16))


def test_merge_projection_full_size(q):
    """The 4096 x 4096 projection weight with its r = 16, alpha = 32 adapter."""
    wl = S.WORKLOADS["c2"]
    d = S.linear_inputs(wl, 0)
    W, A, B = d["W"], d["A"], d["B"]
    N, K = W.shape
    packed, c, _ = nf4.quantize(W)
    e, s2, mu = nf4.double_quant(c)
    W_hat = nf4.dequant(packed, N * K, nf4.dq_constants(e, s2, mu), out="bf16").reshape(N, K)
    merged = lora.merge(W_hat, A.double().numpy(), B.double().numpy(), wl.s)
    _, W_out, codes, absmax = run_merge(q, W, A, B, wl.r, wl.s, True)
    assert np.array_equal(bf16_bits_t(W_out).reshape(-1), F.bf16_bits(merged).reshape(-1))
    packed2, c2, _ = nf4.quantize(merged.reshape(-1))
    assert np.array_equal(np_u8(codes), packed2)
    assert np.array_equal(f32_bits_t(absmax), F.f32_bits(c2))
