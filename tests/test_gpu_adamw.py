"""GPU parity of the fused AdamW step (the paged optimizer's update) against
the oracle's fp32 form (oracle/adamw.py: adamw_step_fp32), bit for bit over
several steps: p, m, v and the bf16 copy of p.  The states live in CUDA
managed memory and are paged out to host memory before every step (the
update pages them back on touch), or prefetched to the device first, or sit in
ordinary device memory; the result must not depend on where the pages were."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import adamw
from oracle import formats as F

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_10_b200 as q
    assert torch.cuda.is_available()
    return q


@pytest.fixture(scope="module")
def rt():
    torch.cuda.init()
    r = ctypes.CDLL("libcudart.so.12")
    r.cudaMallocManaged.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_size_t, ctypes.c_uint]
    r.cudaFree.argtypes = [ctypes.c_void_p]
    return r


def _managed(rt, n):
    ptr = ctypes.c_void_p()
    assert rt.cudaMallocManaged(ctypes.byref(ptr), ctypes.c_size_t(4 * n), 1) == 0
    arr = np.ctypeslib.as_array((ctypes.c_float * n).from_address(ptr.value))
    arr[:] = 0.0
    return ptr.value, arr


@pytest.mark.parametrize("placement", ["host_before_each_step", "device_prefetch", "device_memory"])
@pytest.mark.parametrize("n", [131072 + 17, 3, 2_588_672])
def test_adamw_bit_exact_over_steps(q, rt, placement, n):
    rng = np.random.default_rng(n)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    p = torch.tensor(p0, device="cuda")
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    if placement == "device_memory":
        m_t = torch.zeros(n, dtype=torch.float32, device="cuda")
        v_t = torch.zeros(n, dtype=torch.float32, device="cuda")
        mp, vp = m_t.data_ptr(), v_t.data_ptr()
        read_m, read_v = (lambda: m_t.cpu().numpy()), (lambda: v_t.cpu().numpy())
        owned = []
    else:
        mp, marr = _managed(rt, n)
        vp, varr = _managed(rt, n)
        read_m, read_v = (lambda: marr.copy()), (lambda: varr.copy())
        owned = [mp, vp]
    rp, rm, rv = p0.astype(np.float64), np.zeros(n), np.zeros(n)
    lr, b1, b2, eps, wd = 2e-4, 0.9, 0.999, 1e-8, 0.01
    try:
        for t in range(1, 6):
            g = torch.tensor(rng.standard_normal(n).astype(np.float32), device="cuda")
            if placement == "host_before_each_step":
                q.qlora_paged_prefetch(mp, 4 * n, q.QL_PAGE_HOST)
                q.qlora_paged_prefetch(vp, 4 * n, q.QL_PAGE_HOST)
            elif placement == "device_prefetch":
                q.qlora_paged_prefetch(mp, 4 * n, q.QL_PAGE_DEVICE)
                q.qlora_paged_prefetch(vp, 4 * n, q.QL_PAGE_DEVICE)
            q.qlora_adamw_step(p, g, mp, vp, n, t, lr, b1, b2, eps, wd, p_bf16=pb)
            torch.cuda.synchronize()
            rp, rm, rv = adamw.adamw_step_fp32(rp, g.cpu().double().numpy(), rm, rv, t, lr=lr, b1=b1, b2=b2,
                                               eps=eps, wd=wd)
            assert np.array_equal(p.cpu().numpy().view(np.uint32), F.f32_bits(rp)), t
            assert np.array_equal(read_m().view(np.uint32), F.f32_bits(rm)), t
            assert np.array_equal(read_v().view(np.uint32), F.f32_bits(rv)), t
            assert np.array_equal(pb.cpu().view(torch.int16).numpy().view(np.uint16), F.bf16_bits(F.bf16(rp))), t
        assert q.qlora_get_status() == q.QL_OK
    finally:
        torch.cuda.synchronize()
        for ptr in owned:
            rt.cudaFree(ctypes.c_void_p(ptr))


def test_paged_prefetch_rejects_device_memory(q):
    x = torch.zeros(1024, dtype=torch.float32, device="cuda")
    with pytest.raises(q.QLoraError) as e:
        q.qlora_paged_prefetch(x, 4096, q.QL_PAGE_HOST)
    assert e.value.status == q.QL_ERR_INVALID_ARG
