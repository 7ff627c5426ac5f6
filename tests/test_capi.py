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
    assert lib.status_string(lib.QL_ERR_TIMEOUT) == "device wait timed out"
    for polls in (0, -1, (1 << 20) + 1):
        assert L.qlora_selftest_wait_timeout(polls, s0) == lib.QL_ERR_INVALID_ARG


def test_boundary_calls_document_source_and_errors():
    """Each call of the hot path's boundary cites the passage it restates and
    states its error behaviour in the header comment right above it."""
    text = open(os.path.join(ROOT, "include", "qlora_nf4.h")).read()
    for name in ("nf4_quantize", "nf4_double_quant", "nf4_dequant", "qlora_linear_fwd", "qlora_linear_bwd",
                 "qlora_merge"):
        m = re.search(r"/\*((?:(?!\*/).)*?)\*/\s*(?:#define[^\n]*\n\s*)?ql_status\s+" + name + r"\s*\(", text, flags=re.S)
        assert m, name
        comment = m.group(1)
        assert re.search(r"\[P[1-5]\]", comment), f"{name}: no source citation"
        assert "QL_ERR" in comment, f"{name}: no error behaviour"


@pytest.mark.parametrize("M,N,K,r", [(4096, 4096, 4096, 16), (130, 512, 1024, 16), (1, 28672, 8192, 64),
                                     (600, 384, 320, 8), (16, 256, 512, 8)])
def test_workspace_sizes_follow_the_documented_layout(lib, M, N, K, r):
    """Forward: U [M, r] bf16.  Backward: B^T [r, N], U^T [r, Mp], V [M, r],
    V^T [r, Mp] bf16 (Mp = M rounded up to 8), each piece 256-byte aligned."""
    a256 = lambda b: (b + 255) // 256 * 256
    Mp = (M + 7) // 8 * 8
    assert lib.qlora_workspace_size(lib.QL_OP_FWD, M, N, K, r) == a256(M * r * 2)
    want = a256(r * N * 2) + a256(r * Mp * 2) + a256(M * r * 2) + a256(r * Mp * 2)
    assert lib.qlora_workspace_size(lib.QL_OP_BWD, M, N, K, r) == want
    assert lib.qlora_workspace_size(lib.QL_OP_BWD, M, N, K, 0) == 0
