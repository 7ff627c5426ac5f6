"""Pins for the oracle's codebook, quantizer, double quantization and storage math.

Each test ties the oracle to something other than itself: numbers printed on
the pages (tests/golden/pages_numbers.json), an independent inverse-normal
routine (scipy), library format conversions (torch bf16 / float8_e4m3fn),
exact constructions and brute force on small inputs.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import ndtri

from oracle import formats as F
from oracle import nf4


# ------------------------------------------------------------------ codebook
def test_codebook_shape_from_pages(golden):
    g = golden["codebook_shape"]
    q = nf4.codebook()
    assert q.size == g["levels"]
    assert np.all(np.diff(q) > 0)
    assert (q < 0).sum() == g["negative"] and (q >= 0).sum() == g["non_negative"]
    zero = np.flatnonzero(q == 0.0)
    assert zero.size == 1 and F.f32_bits(q[zero])[0] == 0 and zero[0] == nf4.ZERO_CODE
    assert q[0] == g["min"] and q[-1] == g["max"]


def _halves_with(quantile):
    pos = [0.5 * (quantile(i / 17) + quantile((i + 1) / 17)) for i in range(8, 16)]
    neg = [0.5 * (quantile(i / 19) + quantile((i + 1) / 19)) for i in range(9, 18)]
    return pos, neg


def test_codebook_positive_half_is_page_formula_verbatim():
    # q_i = 1/2 (Q(i/17) + Q((i+1)/17)), i = 8..15, with scipy's ndtri as Q
    pos, _ = _halves_with(lambda p: float(ndtri(p)))
    expect = F.fl32(np.array([0.0] + [v / pos[-1] for v in pos[1:]]))
    assert np.array_equal(F.f32_bits(nf4.codebook()[8:]), F.f32_bits(expect))


def test_codebook_negative_half_independent_quantile():
    _, neg = _halves_with(lambda p: float(ndtri(p)))
    expect = F.fl32(np.array(sorted(-(v / neg[-1]) for v in neg[1:])))
    assert np.array_equal(F.f32_bits(nf4.codebook()[:8]), F.f32_bits(expect))


def test_codebook_values_far_from_fp32_rounding_boundaries():
    # the fp64 quantile error (~1e-16) cannot flip an fp32 rounding
    q64 = nf4.codebook_f64()
    q32 = nf4.codebook()
    ulp = np.spacing(np.abs(q32).astype(np.float32)).astype(np.float64)
    frac = np.abs(q64 - q32) / ulp
    assert np.all(np.abs(frac - 0.5) > 1e-3)


def test_midpoints_between_levels():
    q, m = nf4.codebook(), nf4.midpoints()
    assert m.size == 15
    assert np.all(q[:-1] < m) and np.all(m < q[1:])
    assert m[7] < 0 < m[8]


# -------------------------------------------------------------- formats pins
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    # plant exact ties: low 16 bits = 0x8000
    u = x.view(np.uint32).copy()
    u[:1000] = (u[:1000] & 0xFFFF0000) | 0x8000
    x = u.view(np.float32)
    ours = F.bf16(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_bf16_from_f64_single_rounding_bruteforce():
    rng = np.random.default_rng(6)
    vals = rng.standard_normal(300) * 10.0 ** rng.integers(-5, 5, 300)
    for v in vals:
        r = float(F.bf16(np.array([v]))[0])
        # candidates: the two bf16 neighbours of v (via fp32 truncation and next)
        f = np.float32(v)
        u = int(np.array([f]).view(np.uint32)[0]) & 0xFFFF0000
        cands = []
        for du in (-0x10000, 0, 0x10000, 0x20000):
            cu = (u + du) & 0xFFFFFFFF
            cands.append(float(np.array([cu], dtype=np.uint32).view(np.float32)[0]))
        fv = Fraction(v)
        best = min(cands, key=lambda c: (abs(Fraction(c) - fv),
                                        (int(np.array([np.float32(c)]).view(np.uint32)[0]) >> 16) & 1))
        assert r == best


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]


def test_e4m3_encode_roundtrip_and_torch():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(F.e4m3_encode(F.e4m3_decode(codes)), codes)
    rng = np.random.default_rng(7)
    v = (rng.standard_normal(100000) * 10.0 ** rng.uniform(-3, 2.6, 100000)).astype(np.float32)
    v = v[np.abs(v) <= 448]
    # exact ties between neighbouring E4M3 values
    grid = np.unique(np.abs(F.e4m3_decode(codes)))
    ties = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    v = np.concatenate([v, ties, -ties])
    ours = F.e4m3_encode(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates():
    v = np.array([448.0, 460.0, 463.9, 464.0, 1e6, np.inf, -1e9, -np.inf])
    assert list(F.e4m3_encode(v)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert F.e4m3_encode(np.array([np.nan]))[0] == 0x7F


# ---------------------------------------------------------------- quantizer
def _all_bf16_in(lo, hi):
    u = np.arange(0, 1 << 16, dtype=np.uint32) << 16
    f = u.view(np.float32)
    v = f[np.isfinite(f)].astype(np.float64)
    return v[(v >= lo) & (v <= hi)]


@pytest.mark.parametrize("c", [1.0, 0.0625, 0.078125, 3.5, 2.0 ** -20, 1.7e5])
def test_threshold_codes_equal_nearest_level_bruteforce(c):
    """Every bf16 x in [-c, c]: threshold code == fp64 nearest level of x/c,
    except where x sits within one fp32 ulp of a decision boundary."""
    q = nf4.codebook()
    m = nf4.midpoints()
    xs = _all_bf16_in(-c, c)
    block = np.concatenate([xs, [c]])          # make c the block absmax
    codes = nf4.quantize_codes(block, np.full(-(-block.size // 64), c))[:xs.size]
    nearest = np.argmin(np.abs(xs[:, None] / c - q[None, :]), axis=1)
    bad = np.flatnonzero(codes != nearest)
    for i in bad:
        x = xs[i]
        dist = np.min(np.abs(x - m * c))
        assert dist <= np.spacing(np.float32(abs(x) + 1e-45)) * 2, (x, codes[i], nearest[i])
    assert bad.size <= 8


def test_threshold_tie_goes_to_lower_level():
    m = nf4.midpoints()
    x = np.concatenate([m, [1.0]])             # c = 1 -> t_j = m_j exactly
    codes = nf4.quantize_codes(x, np.array([1.0]))
    assert list(codes[:15]) == list(range(15))


def test_zero_stays_zero_and_special_blocks():
    x = np.zeros(200)
    x[64:128] = np.linspace(-1, 1, 64)
    x[70] = 0.0
    x[71] = -0.0
    codes = nf4.quantize_codes(x)
    assert np.all(codes[:64] == nf4.ZERO_CODE)          # all-zero block
    assert codes[70] == nf4.ZERO_CODE and codes[71] == nf4.ZERO_CODE
    assert codes[64] == 0 and codes[127] == 15          # absmax elements -> endpoints
    assert np.all(codes[128:] == nf4.ZERO_CODE)         # zeros in a partial block


def test_absmax_survives_non_dq_roundtrip():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(64 * 50) * 0.02).astype(np.float32)
    packed, c, _ = nf4.quantize(x)
    w = nf4.dequant(packed, x.size, c, out="f32")
    blocks = np.abs(x.astype(np.float64)).reshape(50, 64)
    i = np.argmax(blocks, axis=1)
    got = np.abs(w.reshape(50, 64)[np.arange(50), i])
    assert np.array_equal(got, c)


@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_roundtrip_idempotence(out):
    rng = np.random.default_rng(2)
    n = 64 * 300 + 37                            # ragged tail
    x = torch.from_numpy((rng.standard_normal(n) * 0.02).astype(np.float32)).to(torch.bfloat16)
    packed, c, _ = nf4.quantize(x)
    codes = nf4.unpack(packed, n)
    w = nf4.dequant(packed, n, c, out=out)
    packed2, c2, _ = nf4.quantize(w)
    assert np.array_equal(nf4.unpack(packed2, n), codes)
    assert np.array_equal(c2, c)


def test_pack_nibble_order_and_odd_tail():
    codes = np.array([1, 2, 3], dtype=np.uint8)
    assert list(nf4.pack(codes)) == [0x21, 0x83]
    assert list(nf4.unpack(nf4.pack(codes), 3)) == [1, 2, 3]


def test_nonfinite_flag():
    x = np.ones(130)
    assert nf4.block_absmax(x)[1]
    x[100] = np.nan
    assert not nf4.block_absmax(x)[1]
    x[100] = np.inf
    assert not nf4.block_absmax(x)[1]


# ------------------------------------------------------- double quantization
def test_tree_sum_order():
    a = np.array([2.0 ** 53, 1.0, 1.0, 1.0, 3.0])
    # ((a0+a1)+(a2+a3)) + (a4+0): fixed adjacent-pair tree, zero padded
    expect = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + 0.0) + (0.0 + 0.0))
    assert nf4.tree_sum_f64(a) == expect
    rng = np.random.default_rng(3)
    b = rng.uniform(0.01, 0.1, 5000).astype(np.float32).astype(np.float64)
    # values in one narrow binade: every partial sum is exact, so any order agrees
    assert nf4.tree_sum_f64(b) == math.fsum(b)


def test_dq_exact_when_constants_on_e4m3_grid():
    """c_b = mu + e_b * s2 with e_b on the E4M3 grid, group max |e| = 448 and
    sum(e) = 0 per group: the reconstruction is bit-exact."""
    rng = np.random.default_rng(4)
    grid = F.e4m3_decode(np.arange(0x00, 0x7F, dtype=np.uint8))   # non-negative finite
    cs = []
    for g, s2 in enumerate([2.0 ** -12, 2.0 ** -11, 2.0 ** -13]):
        half = rng.choice(grid, 127)
        half[0] = 448.0
        e = np.concatenate([half, -half, [0.0, 0.0]])
        rng.shuffle(e)
        cs.append(0.5 + e * s2)
    c = np.concatenate(cs)
    assert np.array_equal(F.fl32(c), c)
    codes, s2, mu = nf4.double_quant(c)
    assert mu == 0.5
    assert list(s2) == [2.0 ** -12, 2.0 ** -11, 2.0 ** -13]
    assert np.array_equal(nf4.dq_constants(codes, s2, mu), c)


def test_dq_constant_absmax_gives_zero_scale():
    c = np.full(600, 0.03125)
    codes, s2, mu = nf4.double_quant(c)
    assert mu == 0.03125 and np.all(s2 == 0) and np.all(codes == 0)
    assert np.all(nf4.dq_constants(codes, s2, mu) == 0.03125)


def test_dq_error_bound_and_group_extreme(golden):
    rng = np.random.default_rng(5)
    g = golden["small_linear_dq_groups"]
    w = (rng.standard_normal(g["N"] * g["K"]) * 0.02).astype(np.float32)
    _, c, _ = nf4.quantize(w)
    assert c.size == g["absmax"]
    codes, s2, mu = nf4.double_quant(c)
    assert s2.size == g["groups"]
    chat = nf4.dq_constants(codes, s2, mu)
    d = F.fl32(c - mu)
    s2b = s2[np.arange(c.size) // 256]
    # E4M3 relative half-ulp 2^-4 (normals), absolute 2^-10 (subnormals), plus fp32 roundings
    bound = s2b * np.maximum(np.abs(d / s2b) * 2.0 ** -4, 2.0 ** -10) + 4 * np.spacing(np.float32(1.0)) * np.abs(c)
    assert np.all(np.abs(chat - c) <= bound)
    # the element with the group's largest |d| codes to +-448
    for k in range(s2.size):
        sl = slice(256 * k, 256 * (k + 1))
        j = np.argmax(np.abs(d[sl]))
        assert codes[sl][j] in (0x7E, 0xFE)


# ------------------------------------------------------------------ storage
def test_storage_arithmetic_matches_pages(golden):
    n = 64 * 256 * 1024
    b_nodq = nf4.storage_bytes(n, dq=False) * 8 / n
    b_dq = (nf4.storage_bytes(n, dq=True) - 4) * 8 / n          # mean amortized away
    assert b_nodq - 4 == golden["scale_overhead_bits_no_dq"]["value"]
    assert b_nodq == golden["bits_per_param_no_dq"]["value"]
    t = golden["dq_overhead_bits"]["terms"]
    assert b_dq - 4 == pytest.approx(t[0] + t[1], abs=1e-5)
    assert round(b_dq - 4, 3) == golden["dq_overhead_bits"]["value"]
    assert round(b_dq, 3) == golden["bits_per_param_dq"]["value"]
    assert round(b_nodq - b_dq, 3) == golden["dq_saving_bits"]["value"]
    assert round(nf4.storage_bytes(n, dq=True) / n, 3) == golden["bytes_per_param_dq"]["value"]
    for key in ("base_weights_8b", "base_weights_14b"):
        p = int(golden[key]["params"])
        assert round(nf4.storage_bytes(p, dq=True) / 2 ** 30, 2) == golden[key]["gb"]
