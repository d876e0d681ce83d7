"""Pins for the QLoRA linear / SwiGLU / chain oracle (``oracle.linear``), independent of the oracle.

Brute force with hand-expanded sums on tiny shapes, the special cases that reduce to a plain layer
(B = 0, s = 0, A = 0), linearity in s, central finite differences of a scalar loss for every gradient,
closed values of silu, and planted mistakes that these pins must catch.
"""

import numpy as np
import pytest

from oracle import linear as L
from oracle import nf4 as O
from qlora_fine_tuning_blockwise_b200 import inputs as I


def tiny(M=3, N=5, K=64, r=2, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    Wd = rng.standard_normal((N, K)) * 0.05
    A = rng.standard_normal((r, K)) * 0.1
    B = rng.standard_normal((N, r)) * 0.1
    dy = rng.standard_normal((M, N))
    return x, Wd, A, B, dy


# ---------------------------------------------------------------------------------------------- brute force


def brute_forward(x, Wd, A, B, s):
    M, K = len(x), len(x[0])
    N, r = len(Wd), len(A)
    y = [[0.0] * N for _ in range(M)]
    for m in range(M):
        u = [sum(x[m][k] * A[j][k] for k in range(K)) for j in range(r)]
        for n in range(N):
            base = sum(x[m][k] * Wd[n][k] for k in range(K))
            lora = sum(u[j] * B[n][j] for j in range(r))
            y[m][n] = base + s * lora
    return np.array(y)


def brute_backward(dy, x, Wd, A, B, s):
    M, K = len(x), len(x[0])
    N, r = len(Wd), len(A)
    v = [[sum(dy[m][n] * B[n][j] for n in range(N)) for j in range(r)] for m in range(M)]
    u = [[sum(x[m][k] * A[j][k] for k in range(K)) for j in range(r)] for m in range(M)]
    dx = [[sum(dy[m][n] * Wd[n][k] for n in range(N)) + s * sum(v[m][j] * A[j][k] for j in range(r))
           for k in range(K)] for m in range(M)]
    dA = [[s * sum(v[m][j] * x[m][k] for m in range(M)) for k in range(K)] for j in range(r)]
    dB = [[s * sum(dy[m][n] * u[m][j] for m in range(M)) for j in range(r)] for n in range(N)]
    return np.array(dx), np.array(dA), np.array(dB)


def test_forward_bruteforce():
    x, Wd, A, B, _ = tiny()
    for s in (2.0, 0.5, -1.25):
        got = L.qlora_forward(x, Wd, A, B, s)
        ref = brute_forward(x.tolist(), Wd.tolist(), A.tolist(), B.tolist(), s)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_backward_bruteforce():
    x, Wd, A, B, dy = tiny(M=4, N=3, r=3)
    got = L.qlora_backward(dy, x, Wd, A, B, 2.0)
    ref = brute_backward(dy.tolist(), x.tolist(), Wd.tolist(), A.tolist(), B.tolist(), 2.0)
    for g, r in zip(got, ref):
        assert g.shape == r.shape
        assert np.allclose(g, r, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------------- special cases


def test_B_zero_reproduces_base_layer_exactly():
    x, Wd, A, B, _ = tiny(M=6, N=7, K=128, r=4)
    y = L.qlora_forward(x, Wd, A, np.zeros_like(B), 2.0)
    assert np.array_equal(y, x @ Wd.T)


def test_s_zero_is_base_layer_and_linear_in_s():
    x, Wd, A, B, _ = tiny(M=6, N=7, K=128, r=4)
    y0 = L.qlora_forward(x, Wd, A, B, 0.0)
    assert np.array_equal(y0, x @ Wd.T)
    y1 = L.qlora_forward(x, Wd, A, B, 1.0)
    y3 = L.qlora_forward(x, Wd, A, B, 3.0)
    assert np.allclose(y3 - y0, 3.0 * (y1 - y0), rtol=1e-12, atol=1e-13)


def test_A_zero_kills_dB_and_lora_part_of_dX():
    x, Wd, A, B, dy = tiny(M=5, N=6, K=64, r=3)
    dx, dA, dB = L.qlora_backward(dy, x, Wd, np.zeros_like(A), B, 2.0)
    assert np.array_equal(dB, np.zeros_like(dB))
    assert np.array_equal(dx, dy @ Wd)
    assert not np.allclose(dA, 0)


def test_quantized_weight_path_uses_dequantized_values():
    """The layer's weight is the NF4 round trip of W (not W itself)."""
    d = I.make_random_linear(8, 16, 128, 4)
    codes, absmax = O.nf4_quantize(d["W"])
    Wd = L.dequantized_weight(codes, absmax, 16, 128)
    assert np.array_equal(Wd.astype(np.float32), O.nf4_dequantize(codes, absmax, 16 * 128).reshape(16, 128))
    assert not np.array_equal(Wd.astype(np.float32), d["W"])


# ---------------------------------------------------------------------------------------------- finite differences


def fd_check(fwd, bwd, x, Wd, A, B, dy, s, h=1e-6, n_probe=12, seed=0):
    """Max relative error between the analytic gradients of L = <dy, y> and central differences."""
    rng = np.random.default_rng(seed)
    dx, dA, dB = bwd(dy, x, Wd, A, B, s)
    worst = 0.0

    def loss(x_, A_, B_):
        return float(np.sum(dy * fwd(x_, Wd, A_, B_, s)))

    for name, arr, grad in (("x", x, dx), ("A", A, dA), ("B", B, dB)):
        for _ in range(n_probe):
            idx = tuple(rng.integers(0, d) for d in arr.shape)
            p, m = arr.copy(), arr.copy()
            p[idx] += h
            m[idx] -= h
            args_p = dict(x_=x, A_=A, B_=B)
            args_m = dict(x_=x, A_=A, B_=B)
            args_p[name + "_"] = p
            args_m[name + "_"] = m
            num = (loss(**args_p) - loss(**args_m)) / (2 * h)
            scale = max(1.0, abs(grad[idx]))
            worst = max(worst, abs(num - grad[idx]) / scale)
    return worst


def test_gradients_match_finite_differences():
    for (M, N, K, r, s) in ((4, 6, 64, 2, 2.0), (3, 5, 64, 4, 0.7), (7, 3, 64, 1, -1.5)):
        x, Wd, A, B, dy = tiny(M, N, K, r, seed=M * 7 + N)
        err = fd_check(L.qlora_forward, L.qlora_backward, x, Wd, A, B, dy, s)
        assert err < 1e-7, err


@pytest.mark.parametrize("mistake", ["drop_s_in_dA", "transpose_in_dB", "sign_in_dx", "drop_lora_in_dx"])
def test_planted_mistakes_are_caught(mistake):
    """A wrong backward planted on the CPU must fail the finite-difference pin."""

    def bad_backward(dy, x, Wd, A, B, s):
        dx, dA, dB = L.qlora_backward(dy, x, Wd, A, B, s)
        if mistake == "drop_s_in_dA":
            dA = dA / s
        elif mistake == "transpose_in_dB":
            dB = (dy.T @ (x @ A.T))[:, ::-1] * s
        elif mistake == "sign_in_dx":
            dx = dy @ Wd - s * ((dy @ B) @ A)
        elif mistake == "drop_lora_in_dx":
            dx = dy @ Wd
        return dx, dA, dB

    x, Wd, A, B, dy = tiny(4, 6, 64, 3)
    assert fd_check(L.qlora_forward, bad_backward, x, Wd, A, B, dy, 2.0, n_probe=30) > 1e-3


# ---------------------------------------------------------------------------------------------- SwiGLU


def test_silu_closed_values():
    assert L.silu(np.array([0.0]))[0] == 0.0
    assert L.silu_grad(np.array([0.0]))[0] == 0.5
    # silu(g) -> g for large g, -> 0 for very negative g
    assert abs(L.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(L.silu(np.array([-40.0]))[0]) < 1e-15
    # silu(1) = 1 / (1 + e^-1)
    assert abs(L.silu(np.array([1.0]))[0] - 1.0 / (1.0 + np.exp(-1.0))) < 1e-16


def test_silu_grad_finite_differences():
    g = np.linspace(-6, 6, 97)
    h = 1e-6
    num = (L.silu(g + h) - L.silu(g - h)) / (2 * h)
    assert np.max(np.abs(num - L.silu_grad(g))) < 1e-8


def test_swiglu_backward_finite_differences():
    rng = np.random.default_rng(1)
    g, u, dh = rng.standard_normal((3, 50))
    dg, du = L.swiglu_backward(dh, g, u)
    h = 1e-6
    num_g = (np.sum(dh * L.swiglu_forward(g + h, u)) - np.sum(dh * L.swiglu_forward(g - h, u)))
    # the loss is a sum of independent terms: probe each coordinate separately
    for i in range(0, 50, 7):
        e = np.zeros(50)
        e[i] = h
        ng = (np.sum(dh * L.swiglu_forward(g + e, u)) - np.sum(dh * L.swiglu_forward(g - e, u))) / (2 * h)
        nu = (np.sum(dh * L.swiglu_forward(g, u + e)) - np.sum(dh * L.swiglu_forward(g, u - e))) / (2 * h)
        assert abs(ng - dg[i]) < 1e-7 and abs(nu - du[i]) < 1e-7
    assert np.isfinite(num_g)


# ---------------------------------------------------------------------------------------------- chain


def test_chain_exact_gradients_finite_differences():
    rng = np.random.default_rng(2)
    M, D, F, r, s = 3, 64, 128, 2, 2.0
    x = rng.standard_normal((M, D))
    mk = lambda n, k: (rng.standard_normal((n, k)) * 0.1, rng.standard_normal((r, k)) * 0.1,
                       rng.standard_normal((n, r)) * 0.1, s)
    gate, up, down = mk(F, D), mk(F, D), mk(D, F)
    dy = rng.standard_normal((M, D))
    y, g, u, h = L.mlp_chain_forward(x, gate, up, down, round_intermediates=False)
    dx, grads = L.mlp_chain_backward(dy, x, gate, up, down, (g, u, h), round_intermediates=False)

    def loss(x_, layers):
        return float(np.sum(dy * L.mlp_chain_forward(x_, *layers, round_intermediates=False)[0]))

    eps = 1e-6
    for idx in ((0, 0), (1, 17), (2, 63)):
        p, m = x.copy(), x.copy()
        p[idx] += eps
        m[idx] -= eps
        num = (loss(p, (gate, up, down)) - loss(m, (gate, up, down))) / (2 * eps)
        assert abs(num - dx[idx]) < 1e-6 * max(1, abs(num))
    for li, name in enumerate(("gate", "up", "down")):
        dA, dB = grads[name]
        for which, grad in ((1, dA), (2, dB)):
            idx = (1, 5) if which == 1 else (5, 1)
            layers = [list(gate), list(up), list(down)]
            base = layers[li][which]
            p, m = base.copy(), base.copy()
            p[idx] += eps
            m[idx] -= eps
            layers[li][which] = p
            lp = loss(x, [tuple(l) for l in layers])
            layers[li][which] = m
            lm = loss(x, [tuple(l) for l in layers])
            num = (lp - lm) / (2 * eps)
            assert abs(num - grad[idx]) < 1e-6 * max(1, abs(num)), (name, which)


def test_chain_rounded_intermediates_are_bf16_and_close_to_exact():
    rng = np.random.default_rng(3)
    M, D, F, r, s = 8, 64, 128, 4, 2.0
    x = O.round_bf16(rng.standard_normal((M, D)).astype(np.float32)).astype(np.float64)
    mk = lambda n, k: (rng.standard_normal((n, k)) * 0.05, rng.standard_normal((r, k)) * 0.1,
                       rng.standard_normal((n, r)) * 0.01, s)
    gate, up, down = mk(F, D), mk(F, D), mk(D, F)
    y, g, u, h = L.mlp_chain_forward(x, gate, up, down, round_intermediates=True)
    for t in (g, u, h):
        assert np.array_equal(O.round_bf16(t.astype(np.float32)).astype(np.float64), t)
    y_exact = L.mlp_chain_forward(x, gate, up, down, round_intermediates=False)[0]
    assert L.compare(y, y_exact)["ok"]


def test_compare_tolerance_semantics():
    ref = np.ones((10, 10))
    assert L.compare(ref * (1 + 5e-3), ref)["ok"]
    assert not L.compare(ref * (1 + 2e-2), ref)["ok"]
    bad = ref.copy()
    bad[0, 0] += 0.05  # one large outlier: Frobenius small, max-abs too large
    assert not L.compare(bad, ref)["ok"]
