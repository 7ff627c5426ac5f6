"""The C-ABI library without a GPU: it loads, exports every function the header
declares, and its host-side helpers and argument checks behave as documented.
No device work is launched here (every call below fails validation first or
is a host helper)."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import formats as F
from oracle import nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z][a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    import bit_nf4_quantized_10_b200._lib as L
    return L


def test_library_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert {"nf4_quantize", "nf4_double_quant", "nf4_dequant", "qlora_linear_fwd", "qlora_linear_bwd"} <= set(declared)
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name


def test_codebook_bitwise_equals_oracle(lib):
    got = np.array(lib.nf4_codebook(), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), F.f32_bits(nf4.codebook()))


@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 16383, 16384, 16385, 64 * 256 * 7 + 5, 8_030_000_000, 4 * 2 ** 30])
def test_storage_bytes_equals_oracle(lib, n):
    assert lib.nf4_storage_bytes(n, True) == nf4.storage_bytes(n, dq=True)
    assert lib.nf4_storage_bytes(n, False) == nf4.storage_bytes(n, dq=False)


def test_workspace_sizes(lib):
    assert lib.qlora_workspace_size(lib.QL_OP_DOUBLE_QUANT, 2048) >= 8
    assert lib.qlora_workspace_size(lib.QL_OP_DOUBLE_QUANT, 64 * 2 ** 20) >= 8 * (2 ** 26 // 2048)
    assert lib.qlora_workspace_size(lib.QL_OP_FWD, 4096, 4096, 4096, 16) >= 4096 * 16 * 2
    assert lib.qlora_workspace_size(lib.QL_OP_FWD, 4096, 4096, 4096, 0) == 0
    assert lib.qlora_workspace_size(lib.QL_OP_BWD, 4096, 4096, 4096, 16) >= 2 * 4096 * 16 * 2
    assert lib.qlora_workspace_size(lib.QL_OP_NVFP4, 100) >= 4


def test_argument_errors_return_before_launch(lib):
    L = lib.LIB
    s0 = ctypes.c_void_p(0)
    fake = 1 << 20                      # aligned, never dereferenced: validation fails first
    assert L.nf4_quantize(None, lib.QL_BF16, 128, fake, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.nf4_quantize(fake + 2, lib.QL_BF16, 128, fake, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.nf4_quantize(fake, 7, 128, fake, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.nf4_quantize(fake, lib.QL_F32, 0, fake, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.nf4_double_quant(fake, 2048, fake, fake, fake, fake, 0, s0) == lib.QL_ERR_WORKSPACE
    assert L.nf4_double_quant(fake, 0, fake, fake, fake, fake, 1 << 20, s0) == lib.QL_ERR_INVALID_ARG
    w = lib.ql_nf4_weight(fake, fake, None, None, None, 256, 500)      # K % 64 != 0
    assert L.qlora_linear_fwd(ctypes.byref(w), fake, 16, fake, fake, 8, 2.0, fake, lib.QL_F32, None, fake,
                              1 << 20, s0) == lib.QL_ERR_INVALID_ARG
    w = lib.ql_nf4_weight(fake, fake, None, None, None, 256, 512)
    assert L.qlora_linear_fwd(ctypes.byref(w), fake, 16, fake, fake, 12, 2.0, fake, lib.QL_F32, None, fake,
                              1 << 20, s0) == lib.QL_ERR_INVALID_ARG                            # r % 8
    assert L.qlora_linear_fwd(ctypes.byref(w), fake, 16, fake, fake, 128, 2.0, fake, lib.QL_F32, None, fake,
                              1 << 20, s0) == lib.QL_ERR_UNSUPPORTED                            # r > 64
    assert L.qlora_linear_fwd(ctypes.byref(w), fake, 16, fake, fake, 8, 2.0, fake, lib.QL_F32, None, fake,
                              0, s0) == lib.QL_ERR_WORKSPACE
    assert L.qlora_linear_bwd(ctypes.byref(w), fake, fake, 16, fake, fake, 8, 2.0, None, fake, lib.QL_F32, 0,
                              fake, fake, lib.QL_F32, fake, 0, s0) == lib.QL_ERR_WORKSPACE
    assert L.nf4_dequant(None, fake, lib.QL_BF16, s0) == lib.QL_ERR_INVALID_ARG
    w = lib.ql_nf4_weight(fake, fake, None, None, None, 256, 500)                           # K % 64 != 0
    assert L.qlora_merge(ctypes.byref(w), fake, fake, 8, 2.0, fake, None, None, s0) == lib.QL_ERR_INVALID_ARG
    w = lib.ql_nf4_weight(fake, fake, None, None, None, 256, 512)
    assert L.qlora_merge(ctypes.byref(w), fake, fake, 8, 2.0, None, None, None, s0) == lib.QL_ERR_INVALID_ARG
    assert L.qlora_merge(ctypes.byref(w), fake, fake, 8, 2.0, None, fake, None, s0) == lib.QL_ERR_INVALID_ARG
    assert L.qlora_merge(ctypes.byref(w), fake, fake, -1, 2.0, fake, None, None, s0) == lib.QL_ERR_INVALID_ARG
    assert L.qlora_merge(ctypes.byref(w), fake, fake, 65, 2.0, fake, None, None, s0) == lib.QL_ERR_UNSUPPORTED
    assert L.qlora_merge(ctypes.byref(w), None, fake, 8, 2.0, fake, None, None, s0) == lib.QL_ERR_INVALID_ARG
    assert L.qlora_merge(ctypes.byref(w), fake, fake, 8, 2.0, fake + 8, None, None, s0) == lib.QL_ERR_INVALID_ARG
    # 4-bit float formats, the AdamW step and the paging helper
    assert L.nvfp4_quantize(fake, lib.QL_BF16, 0, 1, fake, fake, fake, fake, 256, s0) == lib.QL_ERR_INVALID_ARG
    assert L.nvfp4_quantize(fake, lib.QL_BF16, 64, 1, fake, fake, fake, fake, 0, s0) == lib.QL_ERR_WORKSPACE
    assert L.nvfp4_quantize(fake, lib.QL_BF16, 64, 1, fake + 4, fake, fake, fake, 256, s0) == lib.QL_ERR_INVALID_ARG
    assert L.mxfp4_quantize(fake, 9, 64, fake, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.mxfp4_quantize(None, lib.QL_F32, 64, fake, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.nvfp4_dequant(fake, fake, None, 64, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.mxfp4_dequant(fake, fake, -1, fake, s0) == lib.QL_ERR_INVALID_ARG
    adam = lambda n, t, b1, b2, eps, g=fake: L.qlora_adamw_step(fake, g, fake, fake, None, n, t, 1e-3, b1, b2, eps,
                                                                 0.0, s0)
    assert adam(0, 1, 0.9, 0.999, 1e-8) == lib.QL_ERR_INVALID_ARG
    assert adam(16, 0, 0.9, 0.999, 1e-8) == lib.QL_ERR_INVALID_ARG
    assert adam(16, 1, 1.0, 0.999, 1e-8) == lib.QL_ERR_INVALID_ARG
    assert adam(16, 1, 0.9, -0.5, 1e-8) == lib.QL_ERR_INVALID_ARG
    assert adam(16, 1, 0.9, 0.999, -1.0) == lib.QL_ERR_INVALID_ARG
    assert adam(16, 1, 0.9, 0.999, 1e-8, g=fake + 4) == lib.QL_ERR_INVALID_ARG
    g = lambda M, N, K, a=fake, y=fake: L.nvfp4_gemm(a, fake, fake, fake, fake, fake, M, N, K, y, s0)
    assert g(0, 128, 256) == lib.QL_ERR_INVALID_ARG
    assert g(128, 128, 256, a=None) == lib.QL_ERR_INVALID_ARG
    assert g(128, 128, 256, y=fake + 4) == lib.QL_ERR_INVALID_ARG
    assert g(128, 128, 320) == lib.QL_ERR_UNSUPPORTED                                       # K % 256
    assert g(1 << 31, 128, 256) == lib.QL_ERR_UNSUPPORTED
    assert g(128, 1 << 23, 256) == lib.QL_ERR_UNSUPPORTED
    assert L.nvfp4_scale_atoms(fake, 0, 256, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.nvfp4_scale_atoms(fake, 128, 192, fake, s0) == lib.QL_ERR_UNSUPPORTED
    assert L.nvfp4_scale_atoms(fake + 8, 128, 256, fake, s0) == lib.QL_ERR_INVALID_ARG
    mg = lambda M, N, K, a=fake, y=fake: L.mxfp4_gemm(a, fake, fake, fake, M, N, K, y, s0)
    assert mg(128, 0, 256) == lib.QL_ERR_INVALID_ARG
    assert mg(128, 128, 256, a=fake + 2) == lib.QL_ERR_INVALID_ARG
    assert mg(128, 128, 256, y=None) == lib.QL_ERR_INVALID_ARG
    assert mg(128, 128, 384) == lib.QL_ERR_UNSUPPORTED                                      # K % 256
    assert mg(128, 1 << 23, 256) == lib.QL_ERR_UNSUPPORTED
    assert L.mxfp4_scale_atoms(fake, 128, 0, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert L.mxfp4_scale_atoms(fake, 128, 128, fake, s0) == lib.QL_ERR_UNSUPPORTED
    assert L.qlora_paged_prefetch(None, 64, lib.QL_PAGE_HOST, s0) == lib.QL_ERR_INVALID_ARG
    assert L.qlora_paged_prefetch(fake, 0, lib.QL_PAGE_HOST, s0) == lib.QL_ERR_INVALID_ARG
    assert L.qlora_paged_prefetch(fake, 64, 5, s0) == lib.QL_ERR_INVALID_ARG
    assert L.nf4_double_quant_finish(fake, 2, 2048, fake, 2048, fake, fake, fake, fake, 1 << 20,
                                     s0) == lib.QL_ERR_INVALID_ARG     # 2 nodes for 2048 constants
    assert L.nf4_double_quant_level1(fake, 0, fake, s0) == lib.QL_ERR_INVALID_ARG
    assert lib.status_string(lib.QL_ERR_TIMEOUT) == "device wait timed out"
    for polls in (0, -1, (1 << 20) + 1):
        assert L.qlora_selftest_wait_timeout(polls, s0) == lib.QL_ERR_INVALID_ARG


def test_boundary_calls_document_source_and_errors():
    """Each call of the hot path's boundary cites the passage it restates and
    states its error behaviour in the header comment right above it."""
    text = open(os.path.join(ROOT, "include", "qlora_nf4.h")).read()
    for name in ("nf4_quantize", "nf4_double_quant", "nf4_dequant", "qlora_linear_fwd", "qlora_linear_bwd",
                 "qlora_merge", "nvfp4_quantize", "qlora_adamw_step", "nf4_double_quant_level1"):
        m = re.search(r"/\*((?:(?!\*/).)*?)\*/\s*(?:#define[^\n]*\n\s*)*ql_status\s+" + name + r"\s*\(", text, flags=re.S)
        assert m, name
        comment = m.group(1)
        assert re.search(r"\[P[1-5]\]", comment), f"{name}: no source citation"
        assert "QL_ERR" in comment, f"{name}: no error behaviour"


@pytest.mark.parametrize("M,N,K,r", [(4096, 4096, 4096, 16), (130, 512, 1024, 16), (1, 28672, 8192, 64),
                                     (600, 384, 320, 8), (16, 256, 512, 8), (9, 28672, 8192, 16), (8, 1024, 4160, 0)])
def test_workspace_sizes_follow_the_documented_layout(lib, M, N, K, r):
    """Forward: U [M, r] bf16; for 1 <= M <= 16 (the small-token kernels)
    first the fp32 part sums of Y [parts, N, M] and of U [parts, M, r], parts =
    ceil(K / 4096) for M <= 8 and ceil(K / 2048) above.  Backward: B^T [r, N],
    U^T [r, Mp], V [M, r], V^T [r, Mp] bf16 (Mp = M rounded up to 8), each
    piece 256-byte aligned."""
    a256 = lambda b: (b + 255) // 256 * 256
    Mp = (M + 7) // 8 * 8
    if M <= 16:
        parts = -(-K // (4096 if M <= 8 else 2048))
        want_fwd = a256(parts * N * M * 4) + a256(parts * M * max(r, 1) * 4) + a256(M * max(r, 1) * 2)
    else:
        want_fwd = a256(M * r * 2)
    assert lib.qlora_workspace_size(lib.QL_OP_FWD, M, N, K, r) == want_fwd
    want = a256(r * N * 2) + a256(r * Mp * 2) + a256(M * r * 2) + a256(r * Mp * 2)
    assert lib.qlora_workspace_size(lib.QL_OP_BWD, M, N, K, r) == want
    assert lib.qlora_workspace_size(lib.QL_OP_BWD, M, N, K, 0) == 0


def test_nvfp4_scale_atom_sizes(lib):
    """One 512-byte atom per 128-row tile and 64-element block of K."""
    assert lib.nvfp4_scale_atoms_bytes(128, 256) == 4 * 512
    assert lib.nvfp4_scale_atoms_bytes(129, 256) == 2 * 4 * 512       # a partial tile is padded
    assert lib.nvfp4_scale_atoms_bytes(28672, 8192) == 224 * 128 * 512
    assert lib.nvfp4_scale_atoms_bytes(0, 256) == 0


def test_mxfp4_scale_atom_sizes(lib):
    """One 512-byte atom per 128-row tile and 128-element block of K."""
    assert lib.mxfp4_scale_atoms_bytes(128, 256) == 2 * 512
    assert lib.mxfp4_scale_atoms_bytes(300, 512) == 3 * 4 * 512
    assert lib.mxfp4_scale_atoms_bytes(28672, 8192) == 224 * 64 * 512
    assert lib.mxfp4_scale_atoms_bytes(128, 64) == 0
