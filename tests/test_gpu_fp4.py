"""GPU parity of the NVFP4 and MXFP4 block codecs against the oracle
(oracle/fp4.py): packed E2M1 codes, block scales (E4M3 / E8M0), the NVFP4
tensor scale and the dequantized values, bit for bit, on ragged sizes, special
values, exact E2M1 rounding ties, and a 4 Gi-element bf16 tensor (sampled
blocks past element 2^32)."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import fp4
from synthetic import inputs as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


def pack(codes):
    c = np.asarray(codes, dtype=np.uint8)
    n = c.size
    out = np.zeros((n + 1) // 2, dtype=np.uint8)
    out[:] = c[0::2]
    out[: n // 2] |= (c[1::2][: n // 2] << 4).astype(np.uint8)
    return out


def gpu_nvfp4(q, x, use_ts):
    n = x.numel()
    xd = x.cuda()
    codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty((n + 15) // 16, dtype=torch.uint8, device="cuda")
    ts = torch.empty(4, dtype=torch.float32, device="cuda")
    ws = torch.empty(q.qlora_workspace_size(q.QL_OP_NVFP4, n), dtype=torch.uint8, device="cuda")
    q.nvfp4_quantize(xd, codes, scales, ts, ws, use_tensor_scale=use_ts)
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    q.nvfp4_dequant(codes, scales, ts, n, out)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    return codes.cpu().numpy(), scales.cpu().numpy(), ts[:1].cpu().numpy(), out.cpu().numpy()


def gpu_mxfp4(q, x):
    n = x.numel()
    xd = x.cuda()
    codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty((n + 31) // 32, dtype=torch.uint8, device="cuda")
    q.mxfp4_quantize(xd, codes, scales)
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    q.mxfp4_dequant(codes, scales, n, out)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    return codes.cpu().numpy(), scales.cpu().numpy(), out.cpu().numpy()


def check_nvfp4(q, x, use_ts):
    xo = x.double().numpy()
    codes, S_ref, st_ref = fp4.nvfp4_quantize(xo, tensor_scale=use_ts)
    g_codes, g_sc, g_ts, g_out = gpu_nvfp4(q, x, use_ts)
    assert np.array_equal(g_codes, pack(codes)), "NVFP4 codes"
    assert np.array_equal(g_sc, F.e4m3_encode(S_ref).astype(np.uint8)), "E4M3 block scales"
    assert F.f32_bits(g_ts)[0] == F.f32_bits(np.array([st_ref]))[0], "tensor scale"
    ref = fp4.nvfp4_dequant(codes, S_ref, st_ref, xo.size)
    assert np.array_equal(g_out.view(np.uint32), F.f32_bits(ref)), "NVFP4 dequant"


def check_mxfp4(q, x):
    xo = x.double().numpy()
    codes, k = fp4.mxfp4_quantize(xo)
    g_codes, g_sc, g_out = gpu_mxfp4(q, x)
    assert np.array_equal(g_codes, pack(codes)), "MXFP4 codes"
    assert np.array_equal(g_sc.astype(np.int64), np.asarray(k, dtype=np.int64) + 127), "E8M0 scales"
    ref = fp4.mxfp4_dequant(codes, k, xo.size)
    assert np.array_equal(g_out.view(np.uint32), F.f32_bits(ref)), "MXFP4 dequant"


@pytest.mark.parametrize("n", [1, 2, 15, 16, 17, 31, 33, 100, 1029, 64 * 1000 + 13, 1 << 20])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_ragged_sizes(q, n, dtype):
    x = S.normal((n,), 0.02, 4000 + n, dtype=dtype)
    for use_ts in (True, False):
        check_nvfp4(q, x, use_ts)
    check_mxfp4(q, x)


def _special(dtype):
    rng = np.random.default_rng(3)
    parts = [np.zeros(32), -np.zeros(32), np.full(32, 0.015625), rng.standard_normal(32) * 1e-39,   # subnormals
             rng.standard_normal(32) * 1e30, -np.abs(rng.standard_normal(32))]
    # exact E2M1 rounding ties and one fp32 step either side, for several block maxima
    grid = fp4.e2m1_decode(np.arange(8))
    mids = (grid[1:] + grid[:-1]) / 2
    for amax in (6.0, 0.75, 2.0 ** -20, 3.0e3):
        blk = np.concatenate([[amax, -amax], mids * amax / 6, -mids * amax / 6])
        blk = np.concatenate([blk, np.nextafter(blk.astype(np.float32), np.float32(np.inf)),
                              np.nextafter(blk.astype(np.float32), np.float32(-np.inf))]).astype(np.float64)
        parts.append(np.resize(blk, 48))
    x = torch.tensor(np.concatenate(parts), dtype=torch.float32)
    return x.to(dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_special_values_and_ties(q, dtype):
    x = _special(dtype)
    for use_ts in (True, False):
        check_nvfp4(q, x, use_ts)
    check_mxfp4(q, x)


def test_nonfinite_sets_status(q):
    x = S.normal((4096,), 0.02, 8).cuda()
    x[1000] = float("nan")
    codes = torch.empty(2048, dtype=torch.uint8, device="cuda")
    sc16 = torch.empty(256, dtype=torch.uint8, device="cuda")
    sc32 = torch.empty(128, dtype=torch.uint8, device="cuda")
    ts = torch.empty(4, dtype=torch.float32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    q.nvfp4_quantize(x, codes, sc16, ts, ws)
    assert q.qlora_get_status() == q.QL_ERR_NONFINITE
    q.mxfp4_quantize(x, codes, sc32)
    assert q.qlora_get_status() == q.QL_ERR_NONFINITE
    assert q.qlora_get_status() == q.QL_OK


def test_4gi_bf16_sampled(q):
    """4 Gi bf16 elements: sampled 16- and 32-blocks (the first, the last, the
    blocks on both sides of element 2^31) against the oracle; NVFP4's tensor
    scale from the oracle's maximum over the whole tensor."""
    n = 4 * 2 ** 30
    x = S.codec_tensor(n, 0.02, S.seed_of(5, 9, "W"), device="cuda")
    codes = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    sc16 = torch.empty(n // 16, dtype=torch.uint8, device="cuda")
    ts = torch.empty(4, dtype=torch.float32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    q.nvfp4_quantize(x, codes, sc16, ts, ws)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    amax = 0.0
    for s0 in range(0, n, 2 ** 28):
        amax = max(amax, float(np.abs(x[s0:s0 + 2 ** 28].cpu().float().numpy()).max()))
    rng = np.random.default_rng(1)
    nb16 = n // 16
    blocks = np.unique(np.concatenate([rng.integers(0, nb16, 300), [0, nb16 - 1, 2 ** 27 - 1, 2 ** 27, 2 ** 27 + 1]]))
    assert blocks.max() < nb16
    c_dev = codes.cpu().numpy()
    s_dev = sc16.cpu().numpy()
    for b in blocks:
        b = int(b)
        xb = x[16 * b:16 * b + 16].cpu().double().numpy()
        assert xb.size == 16
        # the block followed by a block holding the tensor maximum: the oracle
        # then derives the same tensor scale from its own maximum
        cb, Sb, st = fp4.nvfp4_quantize(np.concatenate([xb, [amax], np.zeros(15)]), tensor_scale=True)
        assert np.array_equal(c_dev[8 * b:8 * b + 8], pack(cb[:16])), b
        assert s_dev[b] == F.e4m3_encode(Sb[:1]).astype(np.uint8)[0], b
    assert F.f32_bits(ts[:1].cpu().numpy())[0] == F.f32_bits(np.array([st]))[0]
    del sc16
    sc32 = torch.empty(n // 32, dtype=torch.uint8, device="cuda")
    q.mxfp4_quantize(x, codes, sc32)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    c_dev = codes.cpu().numpy()
    s_dev = sc32.cpu().numpy()
    nb32 = n // 32
    blocks = np.unique(np.concatenate([rng.integers(0, nb32, 300), [0, nb32 - 1, 2 ** 26 - 1, 2 ** 26, 2 ** 26 + 1]]))
    assert blocks.max() < nb32
    for b in blocks:
        b = int(b)
        xb = x[32 * b:32 * b + 32].cpu().double().numpy()
        assert xb.size == 32
        cb, kb = fp4.mxfp4_quantize(xb)
        assert np.array_equal(c_dev[16 * b:16 * b + 16], pack(cb)), b
        assert int(s_dev[b]) == int(kb[0]) + 127, b
