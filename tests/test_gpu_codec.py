"""GPU parity of the NF4 codec (nf4_quantize, nf4_double_quant, nf4_dequant)
against the oracle: bit-exact codes, packed bytes, fp32 constants, E4M3 codes,
second-level scales, the mean, and the dequantized bf16 / fp32 weights."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import nf4
from synthetic import inputs as S
from tests._parity import np64, np_u8, f32_bits_t, bf16_bits_t

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


def gpu_codec(q, x: torch.Tensor):
    """Quantize a flat device tensor with both constant forms; returns device outputs."""
    xd = x.reshape(1, -1)
    w, absmax = q.quantize_weight(xd, dq=True, keep_absmax=True)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    return w, absmax


def oracle_codec(x):
    packed, c, finite = nf4.quantize(x)
    e, s2, mu = nf4.double_quant(c)
    return packed, c, e, s2, mu


def check_all(q, x_cpu: torch.Tensor):
    n = x_cpu.numel()
    w, absmax = gpu_codec(q, x_cpu.cuda())
    packed, c, e, s2, mu = oracle_codec(x_cpu)
    assert np.array_equal(np_u8(w.codes), packed), "packed codes"
    assert np.array_equal(f32_bits_t(absmax), F.f32_bits(c)), "absmax"
    assert np.array_equal(np_u8(w.absmax_q), e), "E4M3 codes"
    assert np.array_equal(f32_bits_t(w.scale2), F.f32_bits(s2)), "scale2"
    assert f32_bits_t(w.offset)[0] == F.f32_bits(np.array([mu]))[0], "mean"
    chat = nf4.dq_constants(e, s2, mu)
    for dq in (True, False):
        ww = w if dq else q.NF4Weight(1, n, w.codes, absmax=absmax)
        cref = chat if dq else c
        out_b = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        out_f = torch.empty(n, dtype=torch.float32, device="cuda")
        q.nf4_dequant(ww, out_b)
        q.nf4_dequant(ww, out_f)
        torch.cuda.synchronize()
        ref_b = nf4.dequant(packed, n, cref, out="bf16")
        ref_f = nf4.dequant(packed, n, cref, out="f32")
        assert np.array_equal(bf16_bits_t(out_b), F.bf16_bits(ref_b)), f"dequant bf16 dq={dq}"
        assert np.array_equal(f32_bits_t(out_f), F.f32_bits(ref_f)), f"dequant f32 dq={dq}"


def test_small_linear_weight_fp32():
    import bit_nf4_quantized_10_b200 as q
    w = S.WORKLOADS["c1"]
    W = S.linear_inputs(w, 0)["W"]          # 256 x 512 fp32, seed 0
    assert -(-W.numel() // 64) == 2048       # 8 double-quant groups
    check_all(q, W.reshape(-1))


@pytest.mark.parametrize("n", [1, 2, 7, 63, 64, 65, 127, 1000, 64 * 257 + 13, 64 * 256 * 3 + 1])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_ragged_sizes(q, n, dtype):
    x = S.normal((n,), 0.02, 1234 + n, dtype=dtype)
    check_all(q, x)


def test_special_values(q):
    n = 64 * 12 + 5
    x = S.normal((n,), 0.02, 99).clone()
    x[:64] = 0.0                                   # all-zero block
    x[64:128] = -0.0                               # negative zeros
    x[130] = 0.0
    x[131] = -0.0
    x[192:256] = 0.015625                          # constant block (absmax hit many times)
    x[256:320] = torch.tensor(np.ldexp(np.linspace(-1, 1, 64), -140), dtype=torch.float32)  # fp32 subnormals
    x[320:384] = -x[320:384].abs()                 # one-signed block
    x[384:448] *= 1e30                             # huge but finite
    check_all(q, x)


def test_constant_absmax_gives_zero_scale(q):
    x = torch.full((64 * 300,), -0.25, dtype=torch.float32)
    check_all(q, x)


def test_nonfinite_sets_status(q):
    x = S.normal((64 * 10,), 0.02, 5).cuda()
    x[200] = float("nan")
    codes = torch.empty(320, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(10, dtype=torch.float32, device="cuda")
    q.nf4_quantize(x, codes, absmax)
    assert q.qlora_get_status() == q.QL_ERR_NONFINITE
    assert q.qlora_get_status() == q.QL_OK            # read clears it
    x[200] = float("inf")
    q.nf4_quantize(x, codes, absmax)
    assert q.qlora_get_status() == q.QL_ERR_NONFINITE


def test_projection_sized_weight_full(q):
    w = S.WORKLOADS["c2"]
    W = S.linear_inputs(w, 0)["W"]          # 4096 x 4096 fp32
    check_all(q, W.reshape(-1))


def test_codec_4gi_bf16_sampled(q):
    """4 Gi bf16 elements (64-bit indexing): every absmax, E4M3 code, scale and
    the mean bit-exact; packed codes on sampled blocks, including the blocks on
    both sides of element 2^31 (where 32-bit signed indexing would overflow)
    and the last block."""
    n = 4 * 2 ** 30
    x = S.codec_tensor(n, 0.02, S.seed_of(5, 9, "W"), device="cuda")
    w, absmax = gpu_codec(q, x)
    nb = n // 64
    # oracle constants from the input, chunk by chunk
    c = np.empty(nb, dtype=np.float64)
    chunk = 2 ** 28
    for s0 in range(0, n, chunk):
        part = x[s0:s0 + chunk].cpu()
        cc, finite = nf4.block_absmax(part)
        assert finite
        c[s0 // 64:(s0 + chunk) // 64] = cc
    assert np.array_equal(f32_bits_t(absmax), F.f32_bits(c))
    e, s2, mu = nf4.double_quant(c)
    assert f32_bits_t(w.offset)[0] == F.f32_bits(np.array([mu]))[0]
    assert np.array_equal(f32_bits_t(w.scale2), F.f32_bits(s2))
    assert np.array_equal(np_u8(w.absmax_q), e)
    rng = np.random.default_rng(0)
    blocks = np.unique(np.concatenate([rng.integers(0, nb, 200), [0, nb - 1, 2 ** 25 - 1, 2 ** 25, 2 ** 25 + 1]]))
    assert blocks.max() < nb
    codes_dev = w.codes
    for b in blocks:
        b = int(b)
        xb = x[b * 64:(b + 1) * 64].cpu()
        assert xb.numel() == 64
        packed, cb, _ = nf4.quantize(xb)
        assert np.array_equal(np_u8(codes_dev[b * 32:(b + 1) * 32]), packed), b


def _tie_blocks(dtype):
    """Blocks whose elements sit exactly on the decision thresholds
    t_j = fl32(m_j c) and one fp32 step either side, for absmax values from
    fp32-subnormal to near FLT_MAX (both sides of 1e-30)."""
    m = nf4.midpoints().astype(np.float32)
    rng = np.random.default_rng(7)
    mags = [1e-40, 1e-38, 5e-31, 1e-30, 2e-30, 1e-20, 0.0371, 1.0, 3.0, 1e20, 1e37, 3.3e38]
    blocks = []
    for cm in mags:
        for rep in range(3):
            c = np.float32(cm * rng.uniform(0.5, 1.0))
            if dtype == torch.bfloat16:
                c = np.float32(F.bf16(np.array([c]))[0])
            x = (rng.uniform(-1, 1, 64) * c).astype(np.float32)
            x[0], x[1] = c, -c
            t = (m * c).astype(np.float32)
            k = 2
            for tj in t:
                for v in (tj, np.nextafter(tj, np.float32(np.inf)), np.nextafter(tj, np.float32(-np.inf))):
                    if k < 64:
                        x[k] = v
                        k += 1
            blocks.append(x)
    x = torch.from_numpy(np.concatenate(blocks))
    return x.to(dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_threshold_ties_all_magnitudes(q, dtype):
    check_all(q, _tie_blocks(dtype))
