"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies gives up, the kernel returns, QL_ERR_TIMEOUT comes back through
qlora_get_status, and the context stays usable for real work afterwards."""
import time

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import nf4
from synthetic import inputs as S
from tests._parity import np_u8, f32_bits_t

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


def test_bounded_wait_times_out_and_context_survives(q):
    assert q.qlora_get_status() == q.QL_OK
    t0 = time.time()
    q.qlora_selftest_wait_timeout(2000)          # at most ~2 ms of polling
    st = q.qlora_get_status()
    elapsed = time.time() - t0
    assert st == q.QL_ERR_TIMEOUT, q.status_string(st)
    assert elapsed < 5.0
    assert q.qlora_get_status() == q.QL_OK       # reading cleared it
    # the context still runs kernels correctly
    x = S.normal((64 * 40,), 0.02, 3).cuda()
    codes = torch.empty(x.numel() // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(x.numel() // 64, dtype=torch.float32, device="cuda")
    q.nf4_quantize(x, codes, absmax)
    assert q.qlora_get_status() == q.QL_OK
    packed, c, _ = nf4.quantize(x.cpu())
    assert np.array_equal(np_u8(codes), packed)
    assert np.array_equal(f32_bits_t(absmax), F.f32_bits(c))
