"""Pins for the oracle's QLoRA linear and gated-MLP forward/backward.

The matmul library routine is cross-checked by explicit loops; gradients are
checked by central finite differences of <dY, Y> in float64; invariants that
follow from the algebra on the pages (B = 0, alpha = 0) and the page's
adapter-count example are checked directly.
"""
import numpy as np
import pytest

from oracle import formats as F
from oracle import lora, nf4


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_forward_matches_triple_loop():
    rng = np.random.default_rng(0)
    M, N, K, r, s = 3, 5, 4, 2, 1.5
    X, W, A, B = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r)
    Y, U = lora.forward(X, W, A, B, s, materialize=False)
    for m in range(M):
        for n in range(N):
            u = [sum(X[m, k] * A[j, k] for k in range(K)) for j in range(r)]
            y = sum(X[m, k] * W[n, k] for k in range(K)) + s * sum(u[j] * B[n, j] for j in range(r))
            assert Y[m, n] == pytest.approx(y, rel=1e-12, abs=1e-12)


def _fd(f, P, eps=1e-6):
    g = np.zeros_like(P)
    it = np.nditer(P, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = P[i]
        P[i] = old + eps
        fp = f()
        P[i] = old - eps
        fm = f()
        P[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def test_backward_matches_finite_differences():
    rng = np.random.default_rng(1)
    M, N, K, r, s = 4, 6, 5, 3, 0.75
    X, W, A, B, dY = (_rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K),
                      _rand(rng, N, r), _rand(rng, M, N))
    loss = lambda: float(np.sum(dY * lora.forward(X, W, A, B, s, materialize=False)[0]))
    g = lora.backward(X, W, A, B, s, dY, materialize=False)
    for name, P in (("dX", X), ("dA", A), ("dB", B)):
        num = _fd(loss, P)
        assert np.allclose(g[name], num, rtol=1e-8, atol=1e-8), name


def test_invariants_B_zero_and_alpha_zero():
    rng = np.random.default_rng(2)
    M, N, K, r = 4, 6, 5, 3
    X, W, A, dY = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, M, N)
    B0 = np.zeros((N, r))
    Y, _ = lora.forward(X, W, A, B0, 2.0)
    assert np.array_equal(Y, X @ W.T)
    g = lora.backward(X, W, A, B0, 2.0, dY)
    assert np.all(g["dA"] == 0)
    B = _rand(rng, N, r)
    g0 = lora.backward(X, W, A, B, 0.0, dY)
    assert np.all(g0["dA"] == 0) and np.all(g0["dB"] == 0)
    assert np.array_equal(g0["dX"], dY @ W)


def test_adapter_count_from_page(golden):
    g = golden["adapter_params_4096_r16"]
    assert lora.adapter_param_count(g["d"], g["k"], g["r"]) == g["value"]


def test_materialized_U_V_are_bf16():
    rng = np.random.default_rng(3)
    X, W, A, B, dY = (_rand(rng, 4, 8), _rand(rng, 6, 8), _rand(rng, 2, 8),
                      _rand(rng, 6, 2), _rand(rng, 4, 6))
    from oracle.formats import bf16
    _, U = lora.forward(X, W, A, B, 1.0)
    g = lora.backward(X, W, A, B, 1.0, dY)
    assert np.array_equal(U, bf16(X @ A.T)) and np.array_equal(g["V"], bf16(dY @ B))


def test_mlp_backward_matches_finite_differences():
    rng = np.random.default_rng(4)
    M, D, H, r, s = 3, 4, 5, 2, 0.5
    Wg, Wu, Wd = _rand(rng, H, D), _rand(rng, H, D), _rand(rng, D, H)
    Ag, Au, Ad = _rand(rng, r, D), _rand(rng, r, D), _rand(rng, r, H)
    Bg, Bu, Bd = _rand(rng, H, r), _rand(rng, H, r), _rand(rng, D, r)
    X, dy = _rand(rng, M, D), _rand(rng, M, D)
    args = lambda: (X, Wg, Ag, Bg, Wu, Au, Bu, Wd, Ad, Bd, s)
    loss = lambda: float(np.sum(dy * lora.mlp_forward(*args(), materialize=False)["y"]))
    fwd = lora.mlp_forward(*args(), materialize=False)
    g = lora.mlp_backward(*args(), dy, fwd, materialize=False)
    for name, P in (("dX", X), ("dAg", Ag), ("dBg", Bg), ("dAu", Au), ("dBu", Bu),
                    ("dAd", Ad), ("dBd", Bd)):
        assert np.allclose(g[name], _fd(loss, P), rtol=1e-7, atol=1e-8), name


def test_silu_special_values():
    assert lora.silu(np.array([0.0]))[0] == 0.0
    x = np.array([-3.0, 1.0, 20.0])
    assert np.allclose(lora.silu(x), x / (1 + np.exp(-x)), rtol=0, atol=0)


def test_dequant_then_linear_uses_table_values():
    """A weight that is exactly c * q_j quantizes to code j and comes back exact."""
    q = nf4.codebook()
    c = 0.5
    w = np.tile(q * c, 4)[: 64]              # one block: absmax c, every level present
    packed, cb, _ = nf4.quantize(w)
    assert cb[0] == c
    what = nf4.dequant(packed, 64, cb, out="f32")
    assert np.array_equal(what, w)


# ------------------------------------------------------------ adapter merge
def _bf16_inputs(rng, N, K, r, wstd=0.02):
    """A dequantized NF4 weight (bf16 values), and bf16 A, B of the page's scales."""
    import torch
    W = torch.from_numpy((rng.standard_normal((N, K)) * wstd).astype(np.float32))
    packed, c, _ = nf4.quantize(W)
    W_hat = nf4.dequant(packed, N * K, c, out="bf16").reshape(N, K)
    A = F.bf16(rng.uniform(-1.0, 1.0, (r, K)) / np.sqrt(K))
    B = F.bf16(rng.standard_normal((N, r)) * 0.01)
    return W, packed, c, W_hat, A, B


def _ulps(a, b):
    """Distance in bf16 steps between two arrays of bf16 values."""
    def lin(v):
        bits = F.bf16_bits(v).astype(np.int64)
        return np.where(bits & 0x8000, -(bits & 0x7FFF), bits & 0x7FFF)
    return np.abs(lin(a) - lin(b))


def test_merge_zero_adapter_is_the_dequantized_weight():
    rng = np.random.default_rng(11)
    _, _, _, W_hat, A, B = _bf16_inputs(rng, 6, 128, 4)
    assert np.array_equal(lora.merge(W_hat, A, B, 0.0), W_hat)
    assert np.array_equal(lora.merge(W_hat, A, np.zeros_like(B), 2.0), W_hat)


def test_merge_closed_form_on_exact_values():
    # r = 1 and power-of-two entries: every step is exact, W' = W_hat + s b a
    W_hat = np.array([[0.5, -0.25], [0.0, 1.0], [-0.75, 0.125]])
    A = np.array([[0.25, -0.5]])
    B = np.array([[0.125], [-1.0], [0.5]])
    got = lora.merge(W_hat, A, B, 2.0)
    want = W_hat + 2.0 * (B @ A)          # all representable in bf16
    assert np.array_equal(got, want)
    assert got[0, 0] == 0.5625 and got[1, 1] == 2.0


@pytest.mark.parametrize("s", [2.0, 0.75, 0.25])
@pytest.mark.parametrize("r", [1, 8, 16, 64])
def test_merge_within_one_bf16_step_of_the_exact_sum(s, r):
    # W_hat + s B A in exact float64 (errors ~1e-16), rounded once to bf16: the
    # fp32 steps may move a value across a bf16 rounding boundary, nothing more
    rng = np.random.default_rng(100 + r)
    _, _, _, W_hat, A, B = _bf16_inputs(rng, 24, 192, r)
    got = lora.merge(W_hat, A, B, s)
    exact = F.bf16(W_hat + np.float64(np.float32(s)) * (B @ A))
    d = _ulps(got, exact)
    assert d.max() <= 1
    assert (d == 0).mean() > 0.99
    # the update is visible: the merged weight is not the base
    assert (got != W_hat).mean() > 0.5


def test_merge_sign_and_orientation():
    # a mistake in the order of B A (A^T B^T, a transpose) or the sign shows here
    W_hat = np.zeros((2, 3))
    A = np.array([[1.0, 2.0, 4.0]])       # r x K
    B = np.array([[0.5], [-0.25]])        # N x r
    got = lora.merge(W_hat, A, B, 1.0)
    assert np.array_equal(got, np.array([[0.5, 1.0, 2.0], [-0.25, -0.5, -1.0]]))


def test_merge_zero_adapter_requantizes_to_the_original_codes():
    # the merged weight with a zero adapter is the dequantized weight, whose
    # nearest levels are the original codes: re-quantizing gives them back, with
    # constants bf16(c) (the largest level is 1, so the block maximum is bf16(c))
    rng = np.random.default_rng(12)
    N, K = 5, 256
    _, packed, c, W_hat, A, B = _bf16_inputs(rng, N, K, 8)
    merged = lora.merge(W_hat, A, B, 0.0)
    packed2, c2, finite = nf4.quantize(merged.reshape(-1))
    assert finite
    assert np.array_equal(nf4.unpack(packed2, N * K), nf4.unpack(packed, N * K))
    assert np.array_equal(c2, F.bf16(c))


def _bf16_rne(x: float) -> float:
    """Round a Python float to the nearest bf16 value (8 significant bits), ties
    to even: the textbook rule, written out independently of the oracle."""
    import math
    if x == 0.0:
        return x
    m, e = math.frexp(x)            # x = m 2^e, 0.5 <= |m| < 1
    return round(m * 256.0) * 2.0 ** (e - 8)   # Python's round() is ties-to-even


def test_mlp_materialization_points_hand_case():
    """One token, one feature, one hidden unit, zero adapters: every bf16
    materialization point of the gated MLP (g, u, h, dh, dg, du) is checked
    against values worked out by hand from the definition, with weights chosen
    so that leaving out any one rounding (or rounding in a different place)
    changes the value checked."""
    import math
    s = 2.0
    one = np.ones((1, 1))
    zA, zB = np.full((1, 1), 0.5), np.zeros((1, 1))
    wg, wu, wd = 1 + 2.0 ** -9, 3 + 2.0 ** -8, 1 + 3 * 2.0 ** -9
    X, dy = one, one
    args = (X, wg * one, zA, zB, wu * one, zA, zB, wd * one, zA, zB, s)
    f = lora.mlp_forward(*args)
    b = lora.mlp_backward(*args, dy, f)
    sig = lambda t: 1.0 / (1.0 + math.exp(-t))
    g = _bf16_rne(wg)                       # 1 + 2^-9 rounds to 1
    u = _bf16_rne(wu)                       # 3 + 2^-8 rounds to 3
    h = _bf16_rne(g * sig(g) * u)
    dh = _bf16_rne(wd)                      # dy = 1
    dg = _bf16_rne(dh * u * sig(g) * (1 + g * (1 - sig(g))))
    du = _bf16_rne(dh * g * sig(g))
    assert (g, u, h) == (1.0, 3.0, 2.1875)
    assert (dh, du) == (1.0078125, 0.73828125)
    for name, got, want in (("g", f["g"], g), ("u", f["u"], u), ("h", f["h"], h), ("y", f["y"], h * wd),
                            ("dh", b["dh"], dh), ("dg", b["dg"], dg), ("du", b["du"], du),
                            ("dX", b["dX"], dg * wg + du * wu)):
        assert float(np.asarray(got).ravel()[0]) == want, name
    # each rounding matters in this case: without it the checked value moves
    unrounded = {"g": wg, "u": wu, "h": g * sig(g) * u, "dh": wd,
                 "dg": dh * u * sig(g) * (1 + g * (1 - sig(g))), "du": dh * g * sig(g)}
    for name, v in unrounded.items():
        assert v != {"g": g, "u": u, "h": h, "dh": dh, "dg": dg, "du": du}[name], name
    assert _bf16_rne(wg * sig(wg) * u) != h          # silu of the unrounded g
    assert _bf16_rne(wd * u * sig(g) * (1 + g * (1 - sig(g)))) != dg   # the unrounded dh
