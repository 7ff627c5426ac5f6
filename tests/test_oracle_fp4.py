"""Pins for the oracle's MXFP4 / NVFP4 block formats (oracle/fp4.py): the E2M1
grid from the format's fields, rounding checked by brute force over every
candidate value, the MX scale rule, power-of-two invariance, exact blocks and
the error bounds that follow from the grid spacing."""
import numpy as np
import pytest

from oracle import fp4
from oracle import formats as F

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_e2m1_values_from_fields():
    assert np.array_equal(fp4.e2m1_decode(np.arange(8)), GRID)
    assert np.array_equal(fp4.e2m1_decode(np.arange(8, 16)), -GRID)


def _brute_round(v):
    """Nearest of the 15 E2M1 values; a tie goes to the code whose mantissa bit
    is 0; beyond 6 saturate."""
    out = np.empty_like(v)
    for i, x in enumerate(v):
        a = min(abs(x), 6.0)
        d = np.abs(GRID - a)
        best = np.flatnonzero(d == d.min())
        if best.size > 1:                              # a tie: the even code (mantissa bit 0)
            best = [b for b in best if b % 2 == 0]
        out[i] = np.copysign(GRID[best[0]], x)
    return out


def test_e2m1_round_bruteforce():
    rng = np.random.default_rng(0)
    mids = (GRID[1:] + GRID[:-1]) / 2
    v = np.concatenate([rng.uniform(-9, 9, 4000), mids, -mids, GRID, -GRID, [6.5, 7.0, 7.9, 100.0, -7.0]])
    assert np.array_equal(fp4.e2m1_round(v), _brute_round(v))


def test_e2m1_encode_decode_roundtrip():
    rng = np.random.default_rng(1)
    v = rng.uniform(-8, 8, 2000)
    assert np.array_equal(fp4.e2m1_decode(fp4.e2m1_encode(v)), fp4.e2m1_round(v))
    assert fp4.e2m1_encode(np.array([-0.1]))[0] == 8      # -0 keeps its sign bit


def test_mxfp4_scale_rule_and_bounds():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(32 * 500) * np.repeat(np.exp(rng.uniform(-8, 8, 500)), 32)
    codes, k = fp4.mxfp4_quantize(x)
    amax = np.abs(x.reshape(-1, 32)).max(axis=1)
    # the block maximum lands in [4, 8) after scaling
    y = amax / np.ldexp(1.0, k)
    assert np.all((y >= 4) & (y < 8))
    xh = fp4.mxfp4_dequant(codes, k, x.size)
    err = np.abs(xh - x).reshape(-1, 32)
    sc = np.ldexp(1.0, k)[:, None]
    ys = np.abs(x.reshape(-1, 32)) / sc
    assert np.all(err[ys <= 6] <= (sc * np.ones_like(ys))[ys <= 6])      # half the widest step (4 -> 6)
    assert np.all(err <= 2 * sc)                                         # (6, 8) saturates to 6


def test_mxfp4_power_of_two_invariance():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(32 * 64)
    c0, k0 = fp4.mxfp4_quantize(x)
    for j in (-20, -3, 5, 17):
        c, k = fp4.mxfp4_quantize(np.ldexp(x, j))
        assert np.array_equal(c, c0) and np.array_equal(k, k0 + j)


def test_mxfp4_exact_block_and_zero_block():
    vals = np.array([6, -4, 3, 0.5, 0, -1.5, 2, 1] * 4) * 2.0 ** -5
    codes, k = fp4.mxfp4_quantize(vals)
    assert k[0] == -5
    assert np.array_equal(fp4.mxfp4_dequant(codes, k, 32), vals)
    codes, k = fp4.mxfp4_quantize(np.zeros(32))
    assert k[0] == -127 and not codes.any()


@pytest.mark.parametrize("tensor_scale", [False, True])
def test_nvfp4_bounds(tensor_scale):
    rng = np.random.default_rng(4)
    x = rng.standard_normal(16 * 800) * 0.02
    codes, S, s_t = fp4.nvfp4_quantize(x, tensor_scale=tensor_scale)
    # the block scales are E4M3 values
    assert np.array_equal(F.e4m3_round(S), S)
    xh = fp4.nvfp4_dequant(codes, S, s_t, x.size)
    scale = (S * s_t)[:, None]
    err = np.abs(xh - x).reshape(-1, 16)
    amax = np.abs(x.reshape(-1, 16)).max(axis=1, keepdims=True)
    # half the widest step is 1 scale unit; an element beyond 6 units (the scale
    # rounded down) saturates, losing amax - 6 units at most
    assert np.all(err <= np.maximum(scale, amax - 6 * scale) * (1 + 1e-12))
    if tensor_scale:
        # the tensor scale keeps every block scale in E4M3's normal range, where
        # it rounds by at most 2^-4: the saturation loss stays below one unit
        assert S.min() >= 2.0 ** -6 and S.max() <= 448
        assert np.all(err <= scale * (1 + 1e-12))
    else:
        # 0.02-sigma weights put the block scales in E4M3's subnormal range
        assert S.max() < 2.0 ** -6


def test_nvfp4_exact_block():
    S = 0.75 * 2.0 ** -3                         # an E4M3 value; amax = 6 S
    vals = np.array([6, -4, 3, 0.5, 0, -1.5, 2, 1, -6, 4, -3, -0.5, 1.5, -2, -1, 0]) * S
    codes, Sq, s_t = fp4.nvfp4_quantize(vals, tensor_scale=False)
    assert s_t == 1.0 and Sq[0] == S
    assert np.array_equal(fp4.nvfp4_dequant(codes, Sq, s_t, 16), vals)


def test_nvfp4_tensor_scale_power_of_two_invariance():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(16 * 64)
    c0, S0, t0 = fp4.nvfp4_quantize(x)
    c1, S1, t1 = fp4.nvfp4_quantize(np.ldexp(x, -9))
    assert np.array_equal(c0, c1) and np.array_equal(S0, S1) and t1 == np.ldexp(t0, -9)


def test_storage_bits():
    assert fp4.storage_bits_per_element("mxfp4") == 4.25
    assert fp4.storage_bits_per_element("nvfp4") == 4.5


def test_nvfp4_gemm_closed_form():
    """Every element one E2M1 value under one scale: Y = K (v_a S_a s_a)(v_b S_b s_b) exactly."""
    M, N, K = 3, 5, 64
    code_one = fp4.e2m1_encode(np.array([1.5]))[0]        # +1.5
    code_neg = fp4.e2m1_encode(np.array([-3.0]))[0]       # -3
    a = np.full(M * K, code_one, dtype=np.uint8)
    b = np.full(N * K, code_neg, dtype=np.uint8)
    Sa = np.full(M * K // 16, 2.0)
    Sb = np.full(N * K // 16, 0.5)
    Y = fp4.nvfp4_gemm(a, Sa, 0.25, b, Sb, 4.0, M, N, K)
    assert Y.shape == (M, N)
    assert np.all(Y == K * (1.5 * 2.0 * 0.25) * (-3.0 * 0.5 * 4.0))


def test_nvfp4_gemm_exact_rational_bruteforce():
    """A small random case against a sum of exact rationals, element by element:
    the dequantized values are fp32 numbers, so their products and sums are
    exact as fractions; float64 with K = 32 terms is within a few ulp."""
    from fractions import Fraction
    rng = np.random.default_rng(7)
    M, N, K = 4, 3, 32
    xa = rng.standard_normal((M, K))
    xb = rng.standard_normal((N, K)) * 0.02
    ca, Sa, sta = fp4.nvfp4_quantize(xa.reshape(-1))
    cb, Sb, stb = fp4.nvfp4_quantize(xb.reshape(-1))
    Y = fp4.nvfp4_gemm(ca, Sa, sta, cb, Sb, stb, M, N, K)
    A = fp4.nvfp4_dequant(ca, Sa, sta, M * K).reshape(M, K)
    B = fp4.nvfp4_dequant(cb, Sb, stb, N * K).reshape(N, K)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(A[m, k])) * Fraction(float(B[n, k])) for k in range(K))
            assert abs(Fraction(float(Y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 48) + Fraction(1, 2 ** 80)
    # and the dequantized values are the codes times the block scale times the tensor scale
    v = fp4.e2m1_decode(ca).reshape(M, K)
    scale = np.repeat(np.asarray(Sa, dtype=np.float64), 16).reshape(M, K) * sta
    assert np.allclose(A, v * scale, rtol=2 ** -22, atol=0)


def test_mxfp4_gemm_closed_form_per_block_scales():
    """One E2M1 value per operand, a different power-of-two scale on every
    32-element block: Y = sum_b 32 v_a v_b 2^(k_a[b] + k_b[b]) exactly, which
    fails if a block covered 16 elements or the scales of A and B were swapped
    between rows."""
    M, N, K = 2, 3, 128
    va, vb = 1.5, -3.0
    a = np.full(M * K, fp4.e2m1_encode(np.array([va]))[0], dtype=np.uint8)
    b = np.full(N * K, fp4.e2m1_encode(np.array([vb]))[0], dtype=np.uint8)
    ka = np.array([[0, 1, -2, 3], [5, -1, 0, 2]])            # [M, K/32]
    kb = np.array([[1, 0, 0, -3], [2, 2, -4, 0], [0, -1, 1, 1]])
    Y = fp4.mxfp4_gemm(a, ka.reshape(-1), b, kb.reshape(-1), M, N, K)
    for m in range(M):
        for n in range(N):
            want = sum(32 * va * vb * 2.0 ** (ka[m, j] + kb[n, j]) for j in range(K // 32))
            assert Y[m, n] == want


def test_mxfp4_gemm_exact_rational_bruteforce():
    """A small random MXFP4 case against a sum of exact rationals; every
    dequantized value is a dyadic rational, so the bound is a few ulp of
    float64."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    M, N, K = 3, 4, 64
    xa = rng.standard_normal((M, K))
    xb = rng.standard_normal((N, K)) * 0.03
    ca, ka = fp4.mxfp4_quantize(xa.reshape(-1))
    cb, kb = fp4.mxfp4_quantize(xb.reshape(-1))
    Y = fp4.mxfp4_gemm(ca, ka, cb, kb, M, N, K)
    v_a = fp4.e2m1_decode(ca).reshape(M, K)
    v_b = fp4.e2m1_decode(cb).reshape(N, K)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(v_a[m, k])) * Fraction(2) ** int(ka[m * K // 32 + k // 32]) *
                        Fraction(float(v_b[n, k])) * Fraction(2) ** int(kb[n * K // 32 + k // 32]) for k in range(K))
            assert abs(Fraction(float(Y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 48) + Fraction(1, 2 ** 100)
