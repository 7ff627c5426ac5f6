"""nf4_double_quant_noalloc against nf4_double_quant, through the C ABI.

The allocation-free entry point is for callers that cannot allocate device
memory (a plugin handed only tensors and a stream, or code that must not call
cudaMalloc because it may synchronize).  It keeps its scratch in a fixed
array inside the library.  Its outputs must equal the workspace entry point's
bit for bit, on consecutive calls with different inputs (the shared scratch
keeps the previous call's contents and must not leak into the next result).
This file is collected last so a failure here stops a run only after every
other test has run; it also passes run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import nf4
from synthetic import inputs as S

pytestmark = pytest.mark.gpu


def _run_both(q, absmax):
    nb = absmax.numel()
    ng = -(-nb // 256)
    dev = absmax.device
    out = []
    for noalloc in (False, True):
        aq = torch.empty(nb, dtype=torch.uint8, device=dev)
        s2 = torch.empty(ng, dtype=torch.float32, device=dev)
        mu = torch.empty(1, dtype=torch.float32, device=dev)
        if noalloc:
            q.nf4_double_quant_noalloc(absmax, aq, s2, mu)
        else:
            ws = torch.empty(max(16, q.qlora_workspace_size(q.QL_OP_DOUBLE_QUANT, nb)), dtype=torch.uint8, device=dev)
            q.nf4_double_quant(absmax, aq, s2, mu, ws)
        torch.cuda.synchronize()
        out.append((aq.cpu().numpy(), s2.cpu().view(torch.int32).numpy(), mu.cpu().view(torch.int32).numpy()))
    return out


@pytest.mark.parametrize("nb", [1, 2048, 2049, 300_000, 5_000_000])
def test_noalloc_matches_workspace_entry_two_calls(nb):
    import bit_nf4_quantized_10_b200._lib as q
    for call, seed in enumerate((11, 12)):          # two calls in a row, different inputs
        W = S.normal((nb * 64,), 0.02, seed + nb, device="cuda")
        codes = torch.empty(nb * 32, dtype=torch.uint8, device="cuda")
        absmax = torch.empty(nb, dtype=torch.float32, device="cuda")
        q.nf4_quantize(W, codes, absmax)
        (a1, s1, m1), (a2, s2, m2) = _run_both(q, absmax)
        assert np.array_equal(a1, a2), (nb, call)
        assert np.array_equal(s1, s2), (nb, call)
        assert np.array_equal(m1, m2), (nb, call)
    assert q.qlora_get_status() == q.QL_OK


@pytest.mark.parametrize("nb", [2049, 300_000])
def test_noalloc_matches_oracle(nb):
    """The no-allocation entry point against the oracle's double quantization
    directly (mean, E4M3 codes, second-level scales), bit for bit."""
    import bit_nf4_quantized_10_b200._lib as q
    W = S.normal((nb * 64,), 0.02, 31 + nb, device="cuda")
    codes = torch.empty(nb * 32, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(nb, dtype=torch.float32, device="cuda")
    q.nf4_quantize(W, codes, absmax)
    ng = -(-nb // 256)
    aq = torch.empty(nb, dtype=torch.uint8, device="cuda")
    s2 = torch.empty(ng, dtype=torch.float32, device="cuda")
    mu = torch.empty(1, dtype=torch.float32, device="cuda")
    q.nf4_double_quant_noalloc(absmax, aq, s2, mu)
    torch.cuda.synchronize()
    e, s2_ref, mu_ref = nf4.double_quant(absmax.cpu().double().numpy())
    assert np.array_equal(aq.cpu().numpy(), e)
    assert np.array_equal(s2.cpu().view(torch.int32).numpy().view(np.uint32), F.f32_bits(s2_ref))
    assert mu.cpu().view(torch.int32).numpy().view(np.uint32)[0] == F.f32_bits(np.array([mu_ref]))[0]
    assert q.qlora_get_status() == q.QL_OK


def test_noalloc_at_the_maximum_size():
    """nb = QL_NOALLOC_MAX_BLOCKS (64 Mi constants, a 4 Gi-element weight): the
    fixed scratch holds the deepest tree; equal to the workspace entry point."""
    import bit_nf4_quantized_10_b200._lib as q
    nb = 1 << 26
    absmax = S.normal((nb,), 0.02, 77, device="cuda").abs_()
    (a1, s1, m1), (a2, s2, m2) = _run_both(q, absmax)
    assert np.array_equal(a1, a2) and np.array_equal(s1, s2) and np.array_equal(m1, m2)
    assert q.qlora_get_status() == q.QL_OK


def test_noalloc_rejects_oversize_before_launch():
    import bit_nf4_quantized_10_b200._lib as q
    fake = ctypes.c_void_p(1 << 20)
    st = q.LIB.nf4_double_quant_noalloc(fake, (1 << 26) + 1, fake, fake, fake, ctypes.c_void_p(0))
    assert st == q.QL_ERR_UNSUPPORTED
