"""Pins of the fp64 oracle to facts fixed outside the oracle itself.

Each test ties the oracle to something it does not compute the same way:
the page's printed worked example, high-precision decimal arithmetic, a
library ODE solver and a library matrix exponential, closed-form invariants
stated on the pages, and a separately written chunked evaluation.  Together
they catch a dropped term, a wrong sign, lambda = ||k|| instead of ||k||^2,
a transposed readout, a pre-update readout, or an off-by-one in the chunk
algebra.

Passages ("Exact Flow Linear Attention: Exact Solution from Continuous-Time
Dynamics", papernotes.org summary of arXiv 2512.12602, unless noted):
worked example - section 一个完整示例; ODE and Euler step - 关键设计 1;
closed form and Duhamel integral - 关键设计 2; contraction and small-x
expansion - 关键设计 3; expm1 / epsilon clamp - 损失函数 / 训练策略;
readout o_t = S_t^T q_t - flowchart of 整体框架; sub-unit gain - jsqmd.com blog
section 1; RK4 specialisation - jsqmd.com blog section 5.3.
"""
import json
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_d2.json")


def _one(S_prev, k, v, beta, q=None, euler=False):
    """Run the oracle recurrence for a single token on a single state."""
    k = np.asarray(k, float)
    v = np.asarray(v, float)
    S_prev = np.asarray(S_prev, float)
    dk, dv = S_prev.shape
    q = np.zeros(dk) if q is None else np.asarray(q, float)
    o, SL = oracle.recurrence(q.reshape(1, 1, 1, dk), k.reshape(1, 1, 1, dk),
                              v.reshape(1, 1, 1, dv), np.array([[[beta]]]),
                              S_prev.reshape(1, 1, dk, dv), euler=euler, threads=1)
    return o[0, 0, 0], SL[0, 0]


# ---------------------------------------------------------------- worked example
def test_worked_example_printed_values():
    g = json.load(open(GOLDEN))
    p, tol = g["printed"], g["printed_abs_tolerance"]
    a, lam = oracle.gate(np.array([g["k"]]), np.array([g["beta"]]))
    assert lam[0] == p["lambda"]
    assert abs(a[0] - p["alpha"]) < tol
    _, S = _one(g["S_prev"], g["k"], g["v"], g["beta"])
    np.testing.assert_allclose(S, p["S_t"], atol=tol, rtol=0)
    # contraction operator I - alpha k k^T: the state reached with v = 0
    _, S0v = _one(g["S_prev"], g["k"], [0.0, 0.0], g["beta"])
    np.testing.assert_allclose(S0v, p["exact_contraction_operator"], atol=tol, rtol=0)
    # the Euler (DeltaNet) operator I - beta k k^T printed for contrast
    _, Se = _one(g["S_prev"], g["k"], [0.0, 0.0], g["beta"], euler=True)
    np.testing.assert_array_equal(Se, p["euler_contraction_operator"])


def test_worked_example_exact_digits():
    getcontext().prec = 50
    e2 = Decimal(-2).exp()
    alpha = (1 - e2) / 4
    _, S = _one([[1, 0], [0, 1]], [2, 0], [0, 1], 0.5)
    assert abs(S[0, 0] - float(e2)) <= 2e-16
    assert abs(S[0, 1] - float(2 * alpha)) <= 2e-16
    assert S[1, 0] == 0.0 and S[1, 1] == 1.0
    assert abs(oracle.alpha(0.5, 4.0) - float(alpha)) <= 1e-16


# ---------------------------------------------------------------- the gate
@pytest.mark.parametrize("beta", [1e-6, 0.01, 0.3, 0.9, 1.0, 3.0])
@pytest.mark.parametrize("lam", [1e-10, 1e-6, 1e-3, 0.5, 1.0, 4.0, 30.0, 1e4])
def test_gate_matches_decimal(beta, lam):
    """alpha = (1 - e^{-beta*lambda})/lambda evaluated in 50-digit decimal
    arithmetic (no expm1) agrees with the oracle's expm1 form."""
    getcontext().prec = 50
    b, l = Decimal(beta), Decimal(lam)
    ref = (1 - (-(b * l)).exp()) / l
    assert abs(oracle.alpha(beta, lam) - float(ref)) <= 4.5e-16 * float(ref)  # two roundings: expm1 and the division


def test_gate_lambda_zero_limit_and_clamp():
    for beta in [0.0, 1e-3, 0.5, 1.0]:
        assert abs(oracle.alpha(beta, 0.0) - beta) <= 1e-12 * max(beta, 1e-300)
        assert oracle.alpha(beta, 0.0, euler=True) == beta
    # lambda below the 1e-12 clamp: alpha is beta to ~1e-12 relative
    assert abs(oracle.alpha(0.7, 1e-20) - 0.7) < 1e-12
    # k = 0 exactly through the gate: lambda reported unclamped
    a, lam = oracle.gate(np.zeros((3, 4)), np.array([0.2, 0.5, 0.9]))
    assert np.all(lam == 0.0)
    np.testing.assert_allclose(a, [0.2, 0.5, 0.9], rtol=1e-12)


def test_gate_lambda_is_squared_norm():
    rng = np.random.default_rng(0)
    k = rng.standard_normal((5, 7))
    _, lam = oracle.gate(k, np.full(5, 0.5))
    np.testing.assert_allclose(lam, np.linalg.norm(k, axis=1) ** 2, rtol=1e-14)


def test_small_x_expansion_slope_two():
    """|alpha - (beta - beta^2 lambda/2)| = O(beta^3 lambda^2) (关键设计 3)."""
    beta = 0.8
    lams = np.logspace(-4, -1, 7)
    err = np.array([abs(oracle.alpha(beta, l) - (beta - 0.5 * beta * beta * l)) for l in lams])
    slope = np.polyfit(np.log(lams), np.log(err), 1)[0]
    assert 1.9 < slope < 2.1
    # and the leading coefficient is beta^3/6
    np.testing.assert_allclose(err / lams ** 2, beta ** 3 / 6, rtol=0.02)


def test_subunit_gain():
    """0 <= alpha*lambda < 1 and alpha <= beta for beta >= 0 (blog section 1)."""
    for beta in np.linspace(0, 5, 21):
        for lam in np.logspace(-8, 6, 29):
            a = oracle.alpha(beta, lam)
            # strictly below 1 wherever e^{-beta*lambda} is representable next to 1
            assert 0.0 <= a * lam <= 1.0
            assert a * lam < 1.0 or beta * lam > 36.0
            assert a <= beta * (1 + 1e-15)


# ---------------------------------------------------------------- the exact flow
def test_expm_machinery_against_library():
    rng = np.random.default_rng(1)
    for d in (2, 3, 4):
        M = rng.standard_normal((d, d)) * 2.0
        np.testing.assert_allclose(oracle.expm_taylor(M, -1.3), scipy.linalg.expm(-1.3 * M),
                                   rtol=1e-12, atol=1e-13)
    R = np.array([[0.0, -1.0], [1.0, 0.0]])
    t = 2.1
    np.testing.assert_allclose(oracle.expm_taylor(R, t),
                               [[np.cos(t), -np.sin(t)], [np.sin(t), np.cos(t)]], atol=1e-15)


@pytest.mark.parametrize("d", [2, 3, 4])
def test_homogeneous_step_is_matrix_exponential(d):
    """With v = 0 and S_{t-1} = I the oracle step returns e^{-beta k k^T},
    computed here by a brute-force Taylor series that knows nothing of the
    rank-1 collapse (关键设计 2)."""
    rng = np.random.default_rng(10 + d)
    for trial in range(6):
        k = rng.standard_normal(d)
        lam = k @ k
        beta = rng.uniform(0.05, 20.0) / lam
        _, S = _one(np.eye(d), k, np.zeros(d), beta)
        E = oracle.expm_taylor(np.outer(k, k), -beta)
        np.testing.assert_allclose(S, E, rtol=0, atol=1e-13)
        # the brute-force series also agrees with the library exponential
        np.testing.assert_allclose(E, scipy.linalg.expm(-beta * np.outer(k, k)), atol=1e-13)
        # A^2 = lambda A (关键设计 2, rank-1 power identity)
        A = np.outer(k, k)
        np.testing.assert_allclose(A @ A, lam * A, rtol=1e-13)
        np.testing.assert_allclose(np.linalg.matrix_power(A, 4), lam ** 3 * A, rtol=1e-12)


@pytest.mark.parametrize("d,dv", [(2, 2), (3, 2), (4, 3)])
def test_inhomogeneous_step_is_duhamel_integral(d, dv):
    """With S_{t-1} = 0 the oracle step returns int_0^beta e^{-(beta-tau)A} b dtau,
    computed by Gauss-Legendre quadrature of the brute-force exponential."""
    rng = np.random.default_rng(20 + d)
    for trial in range(4):
        k = rng.standard_normal(d)
        v = rng.standard_normal(dv)
        beta = rng.uniform(0.05, 8.0) / (k @ k)
        _, S = _one(np.zeros((d, dv)), k, v, beta)
        Iq = oracle.duhamel(k, v, beta, panels=32)
        np.testing.assert_allclose(S, Iq, rtol=0, atol=1e-12 * np.abs(Iq).max())


def _ode_reference(q, k, v, beta, S0, euler=False):
    """Integrate the piecewise-constant ZOH ODE dS/dtau = -A_t S + b_t over
    tau in [0, beta_t] token by token with scipy's DOP853, reading out
    o_t = S_t^T q_t after each token."""
    L, dk = k.shape
    dv = v.shape[1]
    S = S0.copy()
    os_ = []
    for t in range(L):
        A = np.outer(k[t], k[t])
        b = np.outer(k[t], v[t])
        f = lambda tau, y: (-A @ y.reshape(dk, dv) + b).ravel()
        sol = scipy.integrate.solve_ivp(f, (0.0, beta[t]), S.ravel(), method="DOP853",
                                        rtol=1e-13, atol=1e-15)
        S = sol.y[:, -1].reshape(dk, dv)
        os_.append(S.T @ q[t])
    return np.array(os_), S


@pytest.mark.parametrize("d,dv", [(3, 2), (4, 4)])
def test_multistep_matches_ode_solver(d, dv):
    """Several tokens: the oracle's outputs and final state equal a library
    ODE solver run on the ZOH dynamics (关键设计 1-2) with o_t = S_t^T q_t.
    Pins time order, accumulation, readout orientation and timing."""
    rng = np.random.default_rng(30 + d)
    L = 6
    q = rng.standard_normal((L, d))
    k = rng.standard_normal((L, d))
    v = rng.standard_normal((L, dv))
    beta = rng.uniform(0.1, 1.0, L)
    S0 = rng.standard_normal((d, dv))
    o_ref, S_ref = _ode_reference(q, k, v, beta, S0)
    o, SL = oracle.recurrence(q[None, None], k[None, None], v[None, None], beta[None, None],
                              S0[None, None], threads=1)
    np.testing.assert_allclose(SL[0, 0], S_ref, atol=1e-10)
    np.testing.assert_allclose(o[0, 0], o_ref, atol=1e-10)


def test_euler_mode_is_explicit_euler_step():
    """euler=True is one explicit Euler step of step size beta (关键设计 1)."""
    rng = np.random.default_rng(3)
    d, dv = 4, 3
    for _ in range(5):
        k, v, S = rng.standard_normal(d), rng.standard_normal(dv), rng.standard_normal((d, dv))
        beta = rng.uniform(0, 1)
        f = -np.outer(k, k) @ S + np.outer(k, v)
        _, Se = _one(S, k, v, beta, euler=True)
        np.testing.assert_allclose(Se, S + beta * f, atol=1e-13)


def test_rk4_specialisation_converges_at_fifth_order():
    """One-step error of the RK4 form (blog 5.3) against the oracle's exact
    step falls as beta^5."""
    rng = np.random.default_rng(4)
    d, dv = 3, 2
    k = rng.standard_normal(d)
    v = rng.standard_normal(dv)
    S = rng.standard_normal((d, dv))
    lam = k @ k
    betas = np.logspace(np.log10(0.02), np.log10(0.5), 6) / lam  # above the fp64 floor
    errs = []
    for b in betas:
        _, Sx = _one(S, k, v, b)
        errs.append(np.abs(oracle.rk4_step(k, v, b, S) - Sx).max())
    slope = np.polyfit(np.log(betas), np.log(errs), 1)[0]
    assert 4.7 < slope < 5.3, slope


# ---------------------------------------------------------------- invariants
def test_contraction_along_key():
    """Along k the state scales by exactly e^{-beta lambda}; directions
    orthogonal to k are untouched (关键设计 3)."""
    rng = np.random.default_rng(5)
    d, dv = 6, 4
    for _ in range(5):
        k = rng.standard_normal(d) * rng.uniform(0.1, 3)
        S = rng.standard_normal((d, dv))
        beta = rng.uniform(0, 2)
        lam = k @ k
        _, S1 = _one(S, k, np.zeros(dv), beta)
        np.testing.assert_allclose(k @ S1, np.exp(-beta * lam) * (k @ S), atol=1e-12)
        x = rng.standard_normal(d)
        x -= (x @ k) / lam * k
        np.testing.assert_allclose(x @ S1, x @ S, atol=1e-12)
        v = rng.standard_normal(dv)
        _, S2 = _one(S, k, v, beta)
        np.testing.assert_allclose(k @ S2, np.exp(-beta * lam) * (k @ S) +
                                   (1 - np.exp(-beta * lam)) * v, atol=1e-12)


def test_non_expansive():
    rng = np.random.default_rng(6)
    d, dv, L = 5, 3, 40
    k = rng.standard_normal((L, d)) * 2
    v = rng.standard_normal((L, dv))
    q = rng.standard_normal((L, d))
    beta = rng.uniform(0, 1.5, L)
    S, Sp = rng.standard_normal((d, dv)), rng.standard_normal((d, dv))
    prev = np.linalg.norm(S - Sp, 2)
    for t in range(L):
        _, S = _one(S, k[t], v[t], beta[t], q[t])
        _, Sp = _one(Sp, k[t], v[t], beta[t], q[t])
        cur = np.linalg.norm(S - Sp, 2)
        assert cur <= prev * (1 + 1e-12)
        prev = cur


def test_zero_beta_leaves_state():
    rng = np.random.default_rng(7)
    B, H, L, d = 1, 2, 9, 4
    q, k, v = (rng.standard_normal((B, H, L, d)) for _ in range(3))
    S0 = rng.standard_normal((B, H, d, d))
    o, SL = oracle.recurrence(q, k, v, np.zeros((B, H, L)), S0, threads=1)
    np.testing.assert_array_equal(SL, S0)
    np.testing.assert_allclose(o, np.einsum("bhij,bhti->bhtj", S0, q), atol=1e-14)


def test_split_sequence_chaining():
    """Running L1 tokens then L-L1 tokens from the saved state equals one pass."""
    rng = np.random.default_rng(8)
    B, H, L, d = 2, 1, 23, 5
    q, k, v = (rng.standard_normal((B, H, L, d)) for _ in range(3))
    beta = rng.uniform(0, 1, (B, H, L))
    o, SL = oracle.recurrence(q, k, v, beta, threads=1)
    L1 = 10
    o1, S1 = oracle.recurrence(q[:, :, :L1], k[:, :, :L1], v[:, :, :L1], beta[:, :, :L1], threads=1)
    o2, S2 = oracle.recurrence(q[:, :, L1:], k[:, :, L1:], v[:, :, L1:], beta[:, :, L1:], S1,
                               threads=1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=2), o, atol=1e-13)
    np.testing.assert_allclose(S2, SL, atol=1e-13)


def test_decode_step_is_recurrence_at_length_one():
    rng = np.random.default_rng(9)
    B, H, d = 3, 2, 6
    q, k, v = (rng.standard_normal((B, H, d)) for _ in range(3))
    beta = rng.uniform(0, 1, (B, H))
    S = rng.standard_normal((B, H, d, d))
    o, S1 = oracle.decode_step(q, k, v, beta, S)
    for b in range(B):
        for h in range(H):
            oo, ss = _one(S[b, h], k[b, h], v[b, h], beta[b, h], q[b, h])
            np.testing.assert_array_equal(ss, S1[b, h])
            np.testing.assert_array_equal(oo, o[b, h])


# ---------------------------------------------------------------- chunked form
@pytest.mark.parametrize("C", [1, 7, 16, 64])
@pytest.mark.parametrize("euler", [False, True])
def test_chunked_ut_equals_sequential(C, euler):
    rng = np.random.default_rng(11)
    B, H, L, dk, dv = 2, 2, 150, 8, 6
    q = rng.standard_normal((B, H, L, dk))
    k = rng.standard_normal((B, H, L, dk)) * 0.4
    v = rng.standard_normal((B, H, L, dv))
    beta = rng.uniform(0, 1, (B, H, L))
    S0 = rng.standard_normal((B, H, dk, dv))
    o, SL = oracle.recurrence(q, k, v, beta, S0, euler=euler, threads=2)
    oc, SLc = oracle.chunked(q, k, v, beta, S0, C=C, euler=euler, threads=2)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12 * np.abs(o).max())
    np.testing.assert_allclose(SLc, SL, rtol=0, atol=1e-12 * np.abs(SL).max())


def test_chunked_orthogonal_keys_in_chunk():
    """Mutually orthogonal keys inside a chunk make A = 0 and T = I."""
    d = 8
    Qm, _ = np.linalg.qr(np.random.default_rng(12).standard_normal((d, d)))
    L = 8
    k = (Qm.T * np.linspace(0.5, 2, d)[:, None])[None, None]  # rows orthogonal
    rng = np.random.default_rng(13)
    q = rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    beta = rng.uniform(0, 1, (1, 1, L))
    o, SL = oracle.recurrence(q, k, v, beta, threads=1)
    oc, SLc = oracle.chunked(q, k, v, beta, C=8, threads=1)
    np.testing.assert_allclose(oc, o, atol=1e-13)
    # with orthogonal keys and S0=0 the final state is sum alpha_t k_t v_t^T
    a, _ = oracle.gate(k, beta)
    np.testing.assert_allclose(SL[0, 0], np.einsum("t,ti,tj->ij", a[0, 0], k[0, 0], v[0, 0]),
                               atol=1e-13)
