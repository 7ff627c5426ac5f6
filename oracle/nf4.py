"""NF4 blockwise quantization and double quantization, written out plainly.

TEST INFRASTRUCTURE ONLY (see the package docstring).  float64 numpy with the
roundings of the method made explicit.

Sources:
  [P2] "QLoRA: Quantize Base Weights to 4-Bit", §2.1 (the NF4 quantile formula),
       §2.2 (blocks of 64, fp32 constants; double quantization to 8-bit floats
       in blocks of 256, 0.127 bits per parameter), §4 (0.5 + 0.016 bytes).
  [P3] "QLoRA — Fine-Tuning a 65B Model on One GPU", "Quantization in one
       paragraph" (absmax c = max|x_i|, index of the nearest level to x/c,
       x_hat = c * q_index), "NF4: sixteen levels shaped like the weights"
       (8 negative, 8 non-negative levels with an exact 0, endpoints -1, +1),
       "Double quantization: the constants are not free" (256 fp32 constants
       per group, 8-bit floats, one fp32 second-level constant, mean subtracted
       first).
"""
from __future__ import annotations

from statistics import NormalDist

import numpy as np

from .formats import F64, fl32, bf16, e4m3_encode, e4m3_decode

BLOCK = 64          # [P2] §2.2 B_1 = 64; [P3] "blocks of 64 values"
DQ_GROUP = 256      # [P2] §2.2 B_2 = 256; [P3] "groups 256 of the FP32 constants"
ZERO_CODE = 8       # index of the exact zero level in the table below


# ------------------------------------------------------------------ codebook
def _adjacent_quantile_midpoints(D: int, i_first: int, i_last: int) -> list[float]:
    """[P2] §2.1: q_i = 1/2 (Q_X(i/D) + Q_X((i+1)/D)), Q_X the N(0,1) quantile."""
    Q = NormalDist().inv_cdf
    return [0.5 * (Q(i / D) + Q((i + 1) / D)) for i in range(i_first, i_last + 1)]


def codebook_f64() -> np.ndarray:
    """The 16 NF4 levels in float64, increasing.

    Reading of [P2] §2.1 together with [P3] "NF4: sixteen levels shaped like
    the weights".  The formula with k = 4 (D = 2^k + 1 = 17) has Q(0) = -inf at
    i = 0, so it cannot give all 16 levels as printed.  [P3] fixes the shape: 8
    negative levels, 8 non-negative ones including an exact 0, and endpoints
    exactly -1 and +1.  The plainest reading that meets all of these applies the
    same adjacent-quantile estimator to each half:
      * non-negative half: the formula verbatim, D = 17, i = 8..15.  i = 8
        gives 0, because 8/17 and 9/17 are symmetric about 1/2.  Scale by the
        i = 15 value so the top level is exactly 1.
      * negative half: the same estimator with one more level, D = 19,
        i = 9..17.  i = 9 is again 0.  Drop that 0, mirror the 8 positive
        values, and scale by the largest, so the bottom level is exactly -1.
    """
    pos = _adjacent_quantile_midpoints(17, 8, 15)
    neg = _adjacent_quantile_midpoints(19, 9, 17)
    # the symmetric terms vanish analytically; the float64 quantile routine
    # leaves them at rounding-noise level
    assert abs(pos[0]) < 1e-15 and abs(neg[0]) < 1e-15
    pos[0] = 0.0
    pos = [v / pos[-1] for v in pos]
    negs = [-(v / neg[-1]) for v in neg[1:]]
    levels = sorted(negs) + pos
    return np.array(levels, dtype=F64)


def codebook() -> np.ndarray:
    """The table as stored and used: each level rounded to fp32 (as float64)."""
    return fl32(codebook_f64())


def midpoints() -> np.ndarray:
    """m_j = fl32(fl32(q_j + q_{j+1}) * 0.5), j = 0..14: decision boundaries.

    The fp32 sum is halved exactly (a power-of-two scale of a normal number).
    """
    q = codebook()
    return fl32(fl32(q[:-1] + q[1:]) * 0.5)


# ------------------------------------------------------------------ quantize
def _as_f64_flat(x) -> np.ndarray:
    """Input values as float64 (exact for fp32 and bf16 inputs)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).reshape(-1).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=F64).reshape(-1)


def block_absmax(x) -> tuple[np.ndarray, bool]:
    """c_b = max |x_i| over each block of 64 consecutive elements.

    [P3] "Quantization in one paragraph": one constant per block, the largest
    magnitude in it.  The last block may be partial; its constant covers its
    valid elements only (the pages say nothing about a ragged tail).  Returns
    (c, finite) where finite is False if any element is NaN or +-inf.
    """
    v = _as_f64_flat(x)
    n = v.size
    nb = -(-n // BLOCK)
    pad = np.zeros(nb * BLOCK, dtype=F64)
    pad[:n] = np.abs(v)
    finite = bool(np.all(np.isfinite(v)))
    c = pad.reshape(nb, BLOCK).max(axis=1) if nb else np.zeros(0, dtype=F64)
    return c, finite


def quantize_codes(x, c: np.ndarray | None = None) -> np.ndarray:
    """NF4 code (0..15) of every element.

    [P3]: store the index of the level nearest to x/c.  Reading: nearest is
    decided by comparing x against the fp32 decision thresholds
    t_j = fl32(m_j * c_b), code = #{j : x > t_j}.  Ties go to the lower level.
    No division by c is needed.  This equals the nearest level of x/c except
    within about one fp32 ulp of a midpoint.  A block with c_b = 0 codes every
    element as the zero level ("zero stays zero", [P3]).
    """
    v = _as_f64_flat(x)
    if c is None:
        c, _ = block_absmax(v)
    m = midpoints()
    codes = np.empty(v.size, dtype=np.uint8)
    step = 1 << 20
    for s in range(0, v.size, step):
        xs = v[s:s + step]
        cb = c[np.arange(s, s + xs.size) // BLOCK]
        t = fl32(m[None, :] * cb[:, None])                   # [len, 15]
        code = (xs[:, None] > t).sum(axis=1)
        code = np.where(cb == 0.0, ZERO_CODE, code)
        codes[s:s + xs.size] = code
    return codes


def pack(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: byte k = code[2k] | code[2k+1] << 4.

    An odd count pads the last high nibble with the zero level.
    """
    c = np.asarray(codes, dtype=np.uint8)
    if c.size % 2:
        c = np.concatenate([c, np.array([ZERO_CODE], dtype=np.uint8)])
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def unpack(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out[:n]


def quantize(x):
    """[P3] blockwise absmax quantization: (packed codes, fp32 constants, finite)."""
    c, finite = block_absmax(x)
    codes = quantize_codes(x, c)
    return pack(codes), c, finite


# ---------------------------------------------------------- double quantization
def tree_sum_f64(a: np.ndarray) -> float:
    """Sum in float64 over a fixed adjacent-pair tree.

    Zero-pad to a power of two, then repeat a'[i] = a[2i] + a[2i+1] until one
    value is left.  Writing the order down makes the mean reproducible.
    """
    a = np.asarray(a, dtype=F64)
    if a.size == 0:
        return 0.0
    size = 1
    while size < a.size:
        size *= 2
    t = np.zeros(size, dtype=F64)
    t[:a.size] = a
    while t.size > 1:
        t = t[0::2] + t[1::2]
    return float(t[0])


def double_quant(c: np.ndarray):
    """Quantize the fp32 block constants c_1 to 8-bit floats.

    [P2] §2.2 and [P3] "Double quantization": groups of 256 constants, each
    stored as an 8-bit float, with one fp32 second-level constant per group.
    The mean is subtracted first so the values are centred on zero.
    Readings:
      * One mean per tensor.  The pages' overhead 8/64 + 32/(64*256) bits leaves
        no room for a per-group offset.  mu = fl32(fl64(S / nb)), with S the
        float64 tree sum above.
      * d_b = fl32(c_b - mu).  c_2 = max |d_b| over the group.
        s_2 = fl32(c_2 / 448) maps the group absmax to the largest E4M3 value.
      * e_b = E4M3_rne_satfinite(fl32(d_b / s_2)).  When s_2 == 0 every code
        is 0x00.
      * "8-bit FP8" [P2] vs "8-bit integers" [P4]: E4M3 is taken.
    Returns (codes uint8 [nb], s2 fp32 [ng], mu fp32).
    """
    c = fl32(np.asarray(c, dtype=F64))
    nb = c.size
    mu = float(fl32(tree_sum_f64(c) / nb)) if nb else 0.0
    e, s2 = dq_encode(c, mu)
    return e, s2, mu


def dq_encode(c: np.ndarray, mu: float):
    """The per-group part of double_quant for a given mean: (codes, s2).

    A tensor quantized in shards aligned to groups of 256 constants gets the
    whole tensor's codes when every shard is encoded with the whole tensor's
    mean."""
    c = fl32(np.asarray(c, dtype=F64))
    nb = c.size
    ng = -(-nb // DQ_GROUP)
    d = fl32(c - mu)
    pad = np.zeros(ng * DQ_GROUP, dtype=F64)
    pad[:nb] = np.abs(d)
    c2 = pad.reshape(ng, DQ_GROUP).max(axis=1) if ng else np.zeros(0)
    s2 = fl32(c2 / 448.0)
    s2_b = s2[np.arange(nb) // DQ_GROUP]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = fl32(np.where(s2_b != 0.0, d / np.where(s2_b != 0.0, s2_b, 1.0), 0.0))
    e = e4m3_encode(ratio)
    e = np.where(s2_b == 0.0, 0, e).astype(np.uint8)
    return e, s2


def dq_constants(e: np.ndarray, s2: np.ndarray, mu: float) -> np.ndarray:
    """c_hat_b = fl32(fl32(E4M3(e_b) * s_2) + mu): two roundings, no fused add."""
    e = np.asarray(e, dtype=np.uint8)
    s2_b = np.asarray(s2, dtype=F64)[np.arange(e.size) // DQ_GROUP]
    return fl32(fl32(e4m3_decode(e) * s2_b) + F64(mu))


# -------------------------------------------------------------- dequantization
def dequant(packed, n: int, c: np.ndarray, out: str = "bf16") -> np.ndarray:
    """x_hat = c_b * q_code ([P3] "Quantization in one paragraph").

    fp32 product, then (out="bf16") rounded to bf16, the compute dtype ([P2]
    §3 "Dequantized 16-bit BF16 Weights"; [P3] "Where the gradients actually
    go").  `c` is either the fp32 constants or the double-quant reconstruction
    from dq_constants().
    """
    codes = unpack(packed, n)
    q = codebook()
    cb = np.asarray(c, dtype=F64)[np.arange(n) // BLOCK]
    w = fl32(q[codes] * cb)
    return bf16(w) if out == "bf16" else w


# ------------------------------------------------------------------- storage
def storage_bytes(n: int, dq: bool) -> int:
    """Bytes for n parameters: packed codes plus constants.

    [P2] §2.2 / [P3]: with double quant, one byte per 64-block, one fp32 per
    256 blocks and, by the reading above, one fp32 mean per tensor.  Without it,
    one fp32 per block.
    """
    nb = -(-n // BLOCK)
    ng = -(-nb // DQ_GROUP)
    codes = -(-n // 2)
    return codes + (nb + 4 * ng + 4 if dq else 4 * nb)
