"""4-bit float block formats with per-block scales: MXFP4 and NVFP4 (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).  float64 numpy with the
roundings written out.

Sources:
  [P1] "Lesson 4 of the Finetuning Sessions", "From FP32 to the 4-Bit Horizon":
       MXFP4 (Open Compute Project microscaling): a block of 32 elements shares
       one 8-bit E8M0 scale, always a power of two; NVFP4 (Blackwell): blocks
       of 16 share an 8-bit E4M3 scale, whose 3 mantissa bits allow fractional
       scales.  "From Turing to Blackwell": the 5th-generation tensor cores
       execute these 4-bit tensors natively with the E4M3 scales.

Both formats store E2M1 elements: 1 sign bit, 2 exponent bits (bias 1), 1
mantissa bit; magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no infinities or NaN.

Readings (the pages fix none of these steps):
  - Element rounding: nearest E2M1 value, ties to even (mantissa bit 0),
    magnitudes above 6 saturate to 6.
  - MXFP4 scale: 2^(floor(log2 amax) - 2), the rule of the OCP microscaling
    format: the block's largest magnitude lands in [4, 8), the top binade of
    E2M1 (values in (6, 8) saturate).  An all-zero block takes 2^-127, the
    smallest E8M0 scale.
  - NVFP4 scale: E4M3(amax / 6) per block of 16, round to nearest even,
    saturating at 448, so the largest element maps to about 6.  E4M3 spans
    2^-9 .. 448; with `tensor_scale`, one fp32 scale per tensor, s_t =
    fl32(amax_tensor / (6 * 448)), divides every block scale first and
    multiplies back on dequantization, so the block scales of small weights
    use E4M3's normal range.  A block whose scale rounds to 0 stores zeros.
  - The scale steps are fp32 operations, each rounded once, in this order (a
    kernel takes the same integer decisions):
      denom = fl32(6 s_t),  S = E4M3(fl32(amax_b / denom)),
      scale = fl32(S s_t),  code = E2M1(fl32(x / scale)),
      x_hat = fl32(E2M1(code) scale).

Parity: pinned by tests/test_oracle_fp4.py (E2M1 grid from the format's fields,
brute-force nearest-even rounding, power-of-two scale invariance, exact blocks,
error bounds).
"""
from __future__ import annotations

import numpy as np

from .formats import F64, fl32, e4m3_round, round_to_precision

E2M1_MAX = 6.0
MX_BLOCK = 32       # [P1] "a block of 32 elements shares a single 8-bit scale"
NV_BLOCK = 16       # [P1] "reducing the block size from 32 down to 16 elements"


def e2m1_decode(code) -> np.ndarray:
    """Value of each E2M1 code (0..15) from its fields."""
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    v = np.where(e == 0, m * 0.5, np.ldexp(1.0 + m / 2.0, (e - 1).astype(np.int64)))
    return np.where(s == 1, -v, v).astype(F64)


def e2m1_round(v) -> np.ndarray:
    """Nearest E2M1 value, ties to even, saturating at +-6 (2 significand bits,
    smallest normal exponent 0, subnormal quantum 0.5)."""
    return round_to_precision(v, 2, 0, E2M1_MAX, saturate=True)


def e2m1_encode(v) -> np.ndarray:
    """E2M1 code of e2m1_round(v); -0 keeps its sign bit."""
    r = e2m1_round(v)
    a = np.abs(r)
    table = e2m1_decode(np.arange(8))
    mag = np.searchsorted(table, a)            # exact: a is a table value
    return (mag | (np.signbit(r).astype(np.int64) << 3)).astype(np.uint8)


def _blocks(x, block):
    x = np.asarray(x, dtype=F64).reshape(-1)
    n = x.size
    nb = -(-n // block)
    xb = np.zeros(nb * block, dtype=F64)
    xb[:n] = x
    return xb.reshape(nb, block), n


def mxfp4_quantize(x):
    """(codes uint8 [n], scale exponents int [nb]) of MXFP4 with blocks of 32.

    The scale of block b is 2^k_b, k_b = floor(log2 amax_b) - 2 (2^-127 for an
    all-zero block); each element is e2m1_round(x / 2^k_b)."""
    xb, n = _blocks(x, MX_BLOCK)
    amax = np.abs(xb).max(axis=1)
    with np.errstate(divide="ignore"):
        _, e2 = np.frexp(amax)                  # amax = f 2^e2, f in [0.5, 1)
    k = np.where(amax > 0, e2.astype(np.int64) - 1 - 2, -127)
    k = np.clip(k, -127, 127)
    y = xb / np.ldexp(1.0, k)[:, None]
    codes = e2m1_encode(y).reshape(-1)[:n]
    return codes, k


def mxfp4_dequant(codes, k, n: int) -> np.ndarray:
    v = e2m1_decode(codes)
    return v * np.ldexp(1.0, np.asarray(k, dtype=np.int64)[np.arange(n) // MX_BLOCK])


def nvfp4_quantize(x, tensor_scale: bool = True):
    """(codes uint8 [n], E4M3 block scales as values [nb], fp32 tensor scale).

    s_t = fl32(amax_tensor / 2688) with tensor_scale (2688 = 6 * 448), else 1;
    then the fp32 steps of the module docstring; an element of a block whose
    scale is 0 codes as 0."""
    xb, n = _blocks(x, NV_BLOCK)
    amax_t = float(np.abs(xb).max()) if xb.size else 0.0
    s_t = float(fl32(amax_t / (E2M1_MAX * 448.0))) if tensor_scale and amax_t > 0 else 1.0
    amax = np.abs(xb).max(axis=1)
    denom = fl32(E2M1_MAX * s_t)
    S = e4m3_round(fl32(amax / denom))
    scale = fl32(S * s_t)
    safe = np.where(scale > 0, scale, 1.0)
    y = np.where(scale[:, None] > 0, fl32(xb / safe[:, None]), 0.0)
    codes = e2m1_encode(y).reshape(-1)[:n]
    return codes, S, s_t


def nvfp4_dequant(codes, S, s_t: float, n: int) -> np.ndarray:
    """x_hat = fl32(E2M1(code) fl32(S s_t))."""
    v = e2m1_decode(codes)
    scale = fl32(np.asarray(S, dtype=F64) * F64(s_t))
    return fl32(v * scale[np.arange(n) // NV_BLOCK])


def nvfp4_gemm(a_codes, a_S, a_st: float, b_codes, b_S, b_st: float, M: int, N: int, K: int) -> np.ndarray:
    """Y = A_hat B_hat^T in float64, A [M, K] and B [N, K] row-major NVFP4
    tensors dequantized by nvfp4_dequant.

    [P1] "Lesson 4 of the Finetuning Sessions", "From Turing to Blackwell": the
    5th-generation tensor cores multiply the 4-bit block formats natively, each
    element times its block scale (and the tensor scale), accumulating the
    products.  Reading: the exact value of that product is the product of the
    dequantized tensors; the kernel's fp32 accumulation order is unspecified, so
    parity is within a tolerance."""
    A = nvfp4_dequant(a_codes, a_S, a_st, M * K).reshape(M, K)
    B = nvfp4_dequant(b_codes, b_S, b_st, N * K).reshape(N, K)
    return A @ B.T


def mxfp4_gemm(a_codes, a_k, b_codes, b_k, M: int, N: int, K: int) -> np.ndarray:
    """Y = A_hat B_hat^T in float64, A [M, K] and B [N, K] row-major MXFP4
    tensors dequantized by mxfp4_dequant (block scale exponents a_k, b_k).

    [P1] "Lesson 4 of the Finetuning Sessions", "From Turing to Blackwell", as
    for nvfp4_gemm; "From FP32 to the 4-Bit Horizon": an MXFP4 block scale is a
    power of two and there is no tensor scale, so every product is exact in
    float64 and the result is the product of the dequantized tensors."""
    A = mxfp4_dequant(a_codes, a_k, M * K).reshape(M, K)
    B = mxfp4_dequant(b_codes, b_k, N * K).reshape(N, K)
    return A @ B.T


def storage_bits_per_element(fmt: str) -> float:
    """Bits per element including the block scales (MX: 8 per 32; NV: 8 per 16;
    the single NVFP4 tensor scale is not counted)."""
    return {"mxfp4": 4 + 8 / MX_BLOCK, "nvfp4": 4 + 8 / NV_BLOCK}[fmt]
