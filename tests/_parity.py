"""Comparison helpers shared by the GPU parity tests."""
import numpy as np
import torch

from oracle import formats as F

# Floating-point outputs accumulated in fp32 on the device, against the oracle's
# unrounded float64 result: relative Frobenius error and max-abs error relative
# to the reference's RMS.
REL_FRO = 2e-3
MAX_ABS_RMS = 1e-2


def np64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.uint8)


def f32_bits_t(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int32).numpy().view(np.uint32)


def bf16_bits_t(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def assert_fp_close(got, ref, what="", rel_fro=REL_FRO, max_abs_rms=MAX_ABS_RMS):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    diff = got - ref
    nref = np.linalg.norm(ref)
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    rf = np.linalg.norm(diff) / nref if nref > 0 else np.linalg.norm(diff)
    ma = np.max(np.abs(diff)) if diff.size else 0.0
    assert rf <= rel_fro, f"{what}: rel Frobenius {rf:.3e} > {rel_fro}"
    assert ma <= max_abs_rms * max(rms, 1e-30), f"{what}: max abs {ma:.3e} > {max_abs_rms} * rms {rms:.3e}"
    return rf, ma


def assert_bf16_within_ulp(got_bf16: torch.Tensor, ref64, what="", ulps=1, abs_rms=0.0):
    """Each bf16 output is within `ulps` bf16 ulp of bf16(reference), or within
    abs_rms * rms(reference) of the unrounded reference.

    abs_rms covers outputs that are GEMM results of a bf16 intermediate both
    sides round on their own (V = bf16(dY B) in the backward): a one-ulp
    difference in V moves an output by about 1e-4 * rms, which is many bf16 ulps
    for an output close to zero."""
    ref = np.asarray(ref64, dtype=np.float64)
    ref_r = F.bf16(ref)
    g = bf16_bits_t(got_bf16).astype(np.int64)
    r = F.bf16_bits(ref_r).astype(np.int64)
    # map sign-magnitude bf16 bits onto a monotone integer line
    def lin(b):
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    d = np.abs(lin(g) - lin(r))
    bad = d > ulps
    if abs_rms > 0:
        rms = np.sqrt(np.mean(ref ** 2))
        gv = F.bf16_from_bits(bf16_bits_t(got_bf16)).reshape(ref.shape)
        bad &= np.abs(gv - ref) > abs_rms * rms
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond {ulps} bf16 ulp (max {d.max()})"


def adjoint_bound(s, U, V, *pairs):
    """Allowed |<a1, b1> - <a2, b2>| for identities that hold exactly in real
    arithmetic but whose two sides each use one independently rounded bf16
    copy of U = X A^T or V = dY B (relative rounding <= 2^-8 per element):
    s * 2^-7 * sum|U||V|, plus 1e-5 * sum|a||b| for fp32 accumulation."""
    U, V = np.abs(np.asarray(U, dtype=np.float64)), np.abs(np.asarray(V, dtype=np.float64))
    acc = sum(float(np.abs(a * b).sum()) for a, b in pairs)
    return abs(s) * 2.0 ** -7 * float((U * V).sum()) + 1e-5 * acc


def assert_chain_close(got, ref, bound, what="", rel_fro=REL_FRO):
    """An output that sits after bf16 intermediates each side rounds on its own
    (the MLP chain's g, u, h, dh, dg, du): relative Frobenius error within
    rel_fro, and every element within `bound`, the most a one-ulp difference
    in every bf16 intermediate can move it (2^-7 |intermediate| |weight|
    summed, computed from the oracle's values) plus 1e-5 rms."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), what
    rf = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rf <= rel_fro, f"{what}: rel Frobenius {rf:.3e}"
    rms = np.sqrt(np.mean(ref ** 2))
    excess = np.abs(got - ref) - (bound + 1e-5 * rms)
    assert excess.max() <= 0, f"{what}: {int((excess > 0).sum())} elements beyond the flip bound"
