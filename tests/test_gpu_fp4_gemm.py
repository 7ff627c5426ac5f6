"""GPU parity of the NVFP4 x NVFP4 and MXFP4 x MXFP4 GEMMs on the block-scaled
tensor cores (nvfp4_scale_atoms, nvfp4_gemm, mxfp4_scale_atoms, mxfp4_gemm)
against the oracle: the scale atoms bit for bit against the layout's
definition, Y against oracle.fp4.nvfp4_gemm / mxfp4_gemm (float64 product of
the dequantized operands).  Both sides take the oracle's quantization of the
same seeded inputs."""
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
    if c.size % 2:
        c = np.concatenate([c, np.zeros(1, np.uint8)])
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def atoms_reference(sf, rows, K, vs=16):
    """The scale-atom layout by its definition: [row tile][4 vs-element K block]
    [512 bytes], row m = m0 + 32 m1 and scale kb of the block at byte
    16 m0 + 4 m1 + kb; rows past `rows` are 0."""
    sf = np.asarray(sf, dtype=np.uint8).reshape(rows, K // vs)
    tiles, kblocks = -(-rows // 128), K // (4 * vs)
    out = np.zeros((tiles, kblocks, 512), dtype=np.uint8)
    for t in range(tiles):
        for m in range(128):
            r = t * 128 + m
            if r >= rows:
                continue
            m0, m1 = m % 32, m // 32
            for qb in range(kblocks):
                out[t, qb, 16 * m0 + 4 * m1: 16 * m0 + 4 * m1 + 4] = sf[r, 4 * qb: 4 * qb + 4]
    return out.reshape(-1)


def oracle_operand(x, rows, K):
    """Oracle NVFP4 quantization of a [rows, K] tensor: packed codes, E4M3
    scale bytes (row-major), tensor scale; and the values the oracle keeps."""
    codes, Sv, st = fp4.nvfp4_quantize(x.reshape(-1))
    return pack(codes), F.e4m3_encode(Sv).astype(np.uint8), st, (codes, Sv, st)


def device_operand(q, packed, sf, st, rows, K):
    codes_d = torch.from_numpy(packed).cuda()
    sf_d = torch.from_numpy(sf).cuda()
    atoms = torch.empty(q.nvfp4_scale_atoms_bytes(rows, K), dtype=torch.uint8, device="cuda")
    q.nvfp4_scale_atoms(sf_d, rows, K, atoms)
    ts = torch.tensor([st], dtype=torch.float32, device="cuda")
    return codes_d, atoms, ts


@pytest.mark.parametrize("rows,K", [(128, 256), (200, 512), (1000, 1024)])
def test_scale_atoms_layout(q, rows, K):
    rng = np.random.default_rng(rows + K)
    sf = rng.integers(0, 256, size=rows * K // 16, dtype=np.uint8)
    atoms = torch.empty(q.nvfp4_scale_atoms_bytes(rows, K), dtype=torch.uint8, device="cuda")
    q.nvfp4_scale_atoms(torch.from_numpy(sf).cuda(), rows, K, atoms)
    torch.cuda.synchronize()
    assert np.array_equal(atoms.cpu().numpy(), atoms_reference(sf, rows, K))


SHAPES = [
    # M, N, K
    (128, 128, 256),      # one tile, one stage
    (256, 384, 2048),     # several tiles and stages (the ring wraps)
    (200, 136, 512),      # ragged M and N: partial last tiles
    (64, 1000, 1280),     # M below one tile; N not a multiple of 4
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_nvfp4_gemm_matches_oracle(q, M, N, K):
    xa = S.normal((M, K), 1.0, 900 + M).numpy().astype(np.float64)
    xb = S.normal((N, K), 0.02, 901 + N).numpy().astype(np.float64)
    pa, sfa, sta, ka = oracle_operand(xa, M, K)
    pb, sfb, stb, kb = oracle_operand(xb, N, K)
    a_d, a_atoms, a_ts = device_operand(q, pa, sfa, sta, M, K)
    b_d, b_atoms, b_ts = device_operand(q, pb, sfb, stb, N, K)
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    q.nvfp4_gemm(a_d, a_atoms, a_ts, b_d, b_atoms, b_ts, M, N, K, Y)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    ref = fp4.nvfp4_gemm(*ka, *kb, M, N, K)
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    rms = np.sqrt(np.mean(ref ** 2))
    # exact products, fp32 accumulation: far inside the contract's 2e-3 relative Frobenius
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
    assert np.max(np.abs(got - ref)) <= 1e-4 * rms


def test_nvfp4_gemm_large_sampled_rows(q):
    """2048 tokens x 4096 x 8192 (512 tiles, 32 stages per tile): every output
    of 18 sampled token rows, the first and last among them, against the
    oracle."""
    M, N, K = 2048, 4096, 8192
    xa = S.normal((M, K), 1.0, 950).numpy().astype(np.float64)
    xb = S.normal((N, K), 0.015, 951).numpy().astype(np.float64)
    pa, sfa, sta, ka = oracle_operand(xa, M, K)
    pb, sfb, stb, kb = oracle_operand(xb, N, K)
    a_d, a_atoms, a_ts = device_operand(q, pa, sfa, sta, M, K)
    b_d, b_atoms, b_ts = device_operand(q, pb, sfb, stb, N, K)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q.nvfp4_gemm(a_d, a_atoms, a_ts, b_d, b_atoms, b_ts, M, N, K, Y)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    rows = np.random.default_rng(3).choice(M, 16, replace=False)
    rows = np.concatenate([rows, [0, M - 1]])
    A = fp4.nvfp4_dequant(ka[0], ka[1], ka[2], M * K).reshape(M, K)[rows]
    B = fp4.nvfp4_dequant(kb[0], kb[1], kb[2], N * K).reshape(N, K)
    ref = A @ B.T
    got = Y[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
    assert np.max(np.abs(got - ref)) <= 1e-4 * rms


# ---------------------------------------------------------------- MXFP4 x MXFP4

def mx_operand(q, x, rows, K):
    """Oracle MXFP4 quantization of a [rows, K] tensor, moved to the device with
    its E8M0 scale bytes (k + 127) laid out as atoms; and the oracle's values."""
    codes, k = fp4.mxfp4_quantize(x.reshape(-1))
    sf = (np.asarray(k, dtype=np.int64) + 127).astype(np.uint8)
    atoms = torch.empty(q.mxfp4_scale_atoms_bytes(rows, K), dtype=torch.uint8, device="cuda")
    q.mxfp4_scale_atoms(torch.from_numpy(sf).cuda(), rows, K, atoms)
    return torch.from_numpy(pack(codes)).cuda(), atoms, (codes, k)


@pytest.mark.parametrize("rows,K", [(128, 256), (300, 768), (1000, 1024)])
def test_mxfp4_scale_atoms_layout(q, rows, K):
    rng = np.random.default_rng(rows * 3 + K)
    sf = rng.integers(0, 256, size=rows * K // 32, dtype=np.uint8)
    atoms = torch.empty(q.mxfp4_scale_atoms_bytes(rows, K), dtype=torch.uint8, device="cuda")
    q.mxfp4_scale_atoms(torch.from_numpy(sf).cuda(), rows, K, atoms)
    torch.cuda.synchronize()
    assert np.array_equal(atoms.cpu().numpy(), atoms_reference(sf, rows, K, vs=32))


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_mxfp4_gemm_matches_oracle(q, M, N, K):
    xa = S.normal((M, K), 1.0, 1900 + M).numpy().astype(np.float64)
    xb = S.normal((N, K), 0.02, 1901 + N).numpy().astype(np.float64)
    a_d, a_atoms, ka = mx_operand(q, xa, M, K)
    b_d, b_atoms, kb = mx_operand(q, xb, N, K)
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    q.mxfp4_gemm(a_d, a_atoms, b_d, b_atoms, M, N, K, Y)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    ref = fp4.mxfp4_gemm(*ka, *kb, M, N, K)
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
    assert np.max(np.abs(got - ref)) <= 1e-4 * rms


def test_mxfp4_gemm_wide_exponents(q):
    """Every 32-element block of A scaled by its own power of two between 2^-40
    and 2^40 (B's blocks by the inverse range): the E8M0 scales reach far from
    1, and a block given its neighbour's scale shows at once."""
    M, N, K = 256, 256, 1024
    rng = np.random.default_rng(77)
    ea = rng.integers(-40, 41, size=(M, K // 32))
    eb = rng.integers(-40, 41, size=(N, K // 32))
    xa = S.normal((M, K), 1.0, 1950).numpy().astype(np.float64) * np.repeat(np.ldexp(1.0, ea), 32, axis=1)
    xb = S.normal((N, K), 1.0, 1951).numpy().astype(np.float64) * np.repeat(np.ldexp(1.0, -eb), 32, axis=1)
    a_d, a_atoms, ka = mx_operand(q, xa, M, K)
    b_d, b_atoms, kb = mx_operand(q, xb, N, K)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q.mxfp4_gemm(a_d, a_atoms, b_d, b_atoms, M, N, K, Y)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    ref = fp4.mxfp4_gemm(*ka, *kb, M, N, K)
    got = Y.cpu().numpy().astype(np.float64)
    # terms span 2^-80 .. 2^80: fp32 accumulation keeps the large ones
    assert np.all(np.isfinite(got))
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)


def test_mxfp4_gemm_large_sampled_rows(q):
    """2048 tokens x 4096 x 8192: 18 sampled token rows against the oracle."""
    M, N, K = 2048, 4096, 8192
    xa = S.normal((M, K), 1.0, 1960).numpy().astype(np.float64)
    xb = S.normal((N, K), 0.015, 1961).numpy().astype(np.float64)
    a_d, a_atoms, ka = mx_operand(q, xa, M, K)
    b_d, b_atoms, kb = mx_operand(q, xb, N, K)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q.mxfp4_gemm(a_d, a_atoms, b_d, b_atoms, M, N, K, Y)
    torch.cuda.synchronize()
    assert q.qlora_get_status() == q.QL_OK
    rows = np.random.default_rng(5).choice(M, 16, replace=False)
    rows = np.concatenate([rows, [0, M - 1]])
    A = fp4.mxfp4_dequant(ka[0], ka[1], M * K).reshape(M, K)[rows]
    B = fp4.mxfp4_dequant(kb[0], kb[1], N * K).reshape(N, K)
    ref = A @ B.T
    got = Y[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
    assert np.max(np.abs(got - ref)) <= 1e-4 * rms
