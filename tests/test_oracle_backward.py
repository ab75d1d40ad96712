"""Pins of the fp64 oracle's reverse-mode derivative (the backward pass has
no formula on the pages; it is derived from the recurrence of section
关键设计 2 and checked here against what needs no derivation).

- Central finite differences of the pinned forward oracle, for every input
  element, on tiny problems: exact mode, Euler mode, stiff keys (beta*lambda
  up to 30), near-zero keys (the series branch of d alpha / d lambda) and
  negative beta.
- The gate derivative against its closed form and against finite
  differences across the series/closed-form switch.
- Linearity: the derivative of a loss linear in (o, S_L) is linear in
  (dO, dS_L)."""
import numpy as np
import pytest

import oracle


def _loss(q, k, v, beta, S0, dO, dSL, euler):
    o, S = oracle.recurrence(q, k, v, beta, S0, euler=euler, threads=1)
    return float((o * dO).sum() + (S * dSL).sum())


def _fd_check(q, k, v, beta, S0, euler, h=1e-6, tol=2e-6, seed=0):
    rng = np.random.default_rng(seed)
    dO = rng.standard_normal(v.shape)
    dSL = rng.standard_normal(S0.shape)
    g = oracle.backward(q, k, v, beta, S0, dO, dSL, euler=euler, threads=1)
    names = ("q", "k", "v", "beta", "S0")
    for name, arr, grad in zip(names, (q, k, v, beta, S0), g):
        flat = arr.reshape(-1)
        fd = np.empty_like(flat)
        for i in range(flat.size):
            x0 = flat[i]
            flat[i] = x0 + h
            lp = _loss(q, k, v, beta, S0, dO, dSL, euler)
            flat[i] = x0 - h
            lm = _loss(q, k, v, beta, S0, dO, dSL, euler)
            flat[i] = x0
            fd[i] = (lp - lm) / (2 * h)
        err = np.abs(fd - grad.reshape(-1)).max() / max(1.0, np.abs(fd).max())
        assert err < tol, f"d{name}: finite differences disagree ({err:.2e})"


def _inputs(seed, B=1, H=2, L=7, dk=3, dv=4, knorm=None, beta_lo=0.0, beta_hi=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, L, dk))
    k = rng.standard_normal((B, H, L, dk))
    if knorm is not None:
        k = k / np.linalg.norm(k, axis=-1, keepdims=True) * knorm
    v = rng.standard_normal((B, H, L, dv))
    beta = rng.uniform(beta_lo, beta_hi, (B, H, L))
    S0 = 0.3 * rng.standard_normal((B, H, dk, dv))
    return q, k, v, beta, S0


def test_fd_exact_mode():
    _fd_check(*_inputs(1), euler=False)


def test_fd_euler_mode():
    q, k, v, beta, S0 = _inputs(2)
    _fd_check(q, k * 0.4, v, beta, S0, euler=True)


def test_fd_stiff_keys():
    # beta * lambda up to ~30: alpha saturates at 1/lambda
    _fd_check(*_inputs(3, knorm=5.5), euler=False, h=1e-7, tol=1e-5)


def test_fd_tiny_keys_series_branch():
    # beta * lambda ~ 1e-5: d alpha / d lambda comes from its series
    _fd_check(*_inputs(4, knorm=3e-3), euler=False)


def test_fd_negative_beta():
    _fd_check(*_inputs(5, beta_lo=-0.5, beta_hi=0.5), euler=False)


def test_gate_derivative_matches_finite_differences_across_branches():
    # one token, d = 1, S0 = 0, v = 1: S_L = alpha(beta, k^2) k, so the
    # derivative reduces to the gate's own, on both sides of the switch
    # between the series and the closed form of d alpha / d lambda
    for beta in (0.7, 2.0):
        for lam in (1e-8, 5e-4 / beta, 1e-3 / beta, 2e-3 / beta, 1.0, 30.0):
            kk = np.sqrt(lam)
            q = np.array([[[[1.0]]]]); k = np.array([[[[kk]]]]); v = np.array([[[[1.0]]]])
            b = np.array([[[beta]]]); S0 = np.zeros((1, 1, 1, 1))
            dO = np.zeros((1, 1, 1, 1)); dSL = np.ones((1, 1, 1, 1))
            _, dk_, _, db, _ = oracle.backward(q, k, v, b, S0, dO, dSL, threads=1)
            # d alpha / d beta = e^{-beta lambda} in closed form (finite
            # differences of the saturated alpha are noise-dominated)
            assert db[0, 0, 0] == pytest.approx(np.exp(-beta * max(lam, 1e-12)) * kk, rel=1e-12), (beta, lam)
            hk = 1e-6 * kk
            f = lambda x: oracle.alpha(beta, x * x) * x
            dk_fd = (f(kk + hk) - f(kk - hk)) / (2 * hk)
            assert dk_[0, 0, 0, 0] == pytest.approx(dk_fd, rel=1e-6, abs=1e-12), (beta, lam)


def test_backward_is_linear_in_the_cotangents():
    q, k, v, beta, S0 = _inputs(6)
    rng = np.random.default_rng(9)
    dO1, dO2 = rng.standard_normal(v.shape), rng.standard_normal(v.shape)
    dS1, dS2 = rng.standard_normal(S0.shape), rng.standard_normal(S0.shape)
    g1 = oracle.backward(q, k, v, beta, S0, dO1, dS1, threads=1)
    g2 = oracle.backward(q, k, v, beta, S0, dO2, dS2, threads=1)
    g12 = oracle.backward(q, k, v, beta, S0, dO1 + 2 * dO2, dS1 + 2 * dS2, threads=1)
    for a, b, c in zip(g1, g2, g12):
        np.testing.assert_allclose(c, a + 2 * b, rtol=1e-12, atol=1e-12)
