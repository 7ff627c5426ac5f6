"""Pins for the oracle's AdamW step (oracle/adamw.py): closed forms of the first
step, weight decay alone, zero gradients, and agreement with torch.optim.AdamW
(an independent library routine) over several steps."""
import numpy as np
import torch

from oracle import adamw


def test_first_step_moves_by_lr_times_sign():
    # t = 1: mhat = g, vhat = g^2, so with eps = 0 the step is lr * g / |g| = lr sign(g)
    rng = np.random.default_rng(0)
    p = rng.standard_normal(1000)
    g = rng.standard_normal(1000)
    p1, m, v = adamw.adamw_step(p, g, np.zeros(1000), np.zeros(1000), 1, lr=1e-3, eps=0.0)
    assert np.allclose(p1, p - 1e-3 * np.sign(g), rtol=0, atol=1e-15)
    assert np.allclose(m, 0.1 * g) and np.allclose(v, 0.001 * g * g)


def test_weight_decay_alone_and_zero_gradient():
    p = np.array([1.0, -2.0, 0.5])
    z = np.zeros(3)
    p1, m, v = adamw.adamw_step(p, z, z, z, 1, lr=0.01, wd=0.1)
    assert np.allclose(p1, p * (1 - 0.01 * 0.1), rtol=0, atol=1e-15)
    assert not m.any() and not v.any()


def test_matches_torch_adamw_over_steps():
    rng = np.random.default_rng(1)
    p0 = rng.standard_normal((16, 64))
    grads = [rng.standard_normal((16, 64)) for _ in range(5)]
    lr, b1, b2, eps, wd = 2e-4, 0.9, 0.999, 1e-8, 0.01
    tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([tp], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = adamw.adamw_step(p, g, m, v, t, lr=lr, b1=b1, b2=b2, eps=eps, wd=wd)
    assert np.allclose(p, tp.detach().numpy(), rtol=0, atol=1e-14)


def test_fp32_form_tracks_the_float64_update():
    # the fp32 step differs from the float64 one only by fp32 roundings
    rng = np.random.default_rng(2)
    p0 = rng.standard_normal(4096).astype(np.float32).astype(np.float64)
    p, m, v = p0.copy(), np.zeros(4096), np.zeros(4096)
    q, mq, vq = p0.copy(), np.zeros(4096), np.zeros(4096)
    for t in range(1, 6):
        g = rng.standard_normal(4096).astype(np.float32).astype(np.float64)
        p, m, v = adamw.adamw_step(p, g, m, v, t, lr=1e-3, wd=0.01)
        q, mq, vq = adamw.adamw_step_fp32(q, g, mq, vq, t, lr=1e-3, wd=0.01)
    assert np.all(q == q.astype(np.float32).astype(np.float64))      # fp32 values
    assert np.max(np.abs(q - p)) < 5 * 2.0 ** -24 * np.max(np.abs(p))
    # the fp32 betas differ from the float64 ones by ~1e-8; m can cancel to near
    # zero, so its error is measured against its scale
    assert np.max(np.abs(mq - m)) < 1e-6 * np.max(np.abs(m))


def test_fp32_form_first_step_is_plus_minus_lr_when_eps_is_zero():
    rng = np.random.default_rng(3)
    p = np.zeros(256)
    g = rng.standard_normal(256).astype(np.float32).astype(np.float64)
    q, _, _ = adamw.adamw_step_fp32(p, g, np.zeros(256), np.zeros(256), 1, lr=0.5, eps=0.0)
    # m / c1 = g (1 - b1 and 1 - b1^1 are the same fp32 number) and sqrt(v / c2) = |g|
    # up to a few roundings, so the step is 0.5 to within a few fp32 ulps
    assert np.allclose(np.abs(q), 0.5, rtol=8 * 2.0 ** -24, atol=0)
    assert np.array_equal(np.sign(q), -np.sign(g))
