"""efla_prefill_bwd on the GPU against the fp64 oracle's reverse-mode
derivative (itself pinned by finite differences in test_oracle_backward.py).

The kernel computes in fp32 throughout (bf16 inputs are exact in fp32), so
every gradient is held to the fp32 bar: max|err| <= 1e-4 * max|ref|."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def efla():
    import delta_rule_linear_03_b200 as m
    return m


def _case(name, B, H, L, seed=0, S0=True, dSL=True, euler=False, kscale=None):
    x = workloads.chunk_inputs(name, B=B, H=H, L=L)
    if kscale is not None:
        x["k"] = (x["k"].float() * kscale).to(x["k"].dtype)
    d = x["k"].shape[-1]
    rng = np.random.default_rng(seed)
    dO = torch.from_numpy(rng.standard_normal((B, H, L, d)).astype(np.float32))
    dS = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32)) if dSL else None
    s0 = workloads.random_state(B, H, d, seed=seed + 1) if S0 else None
    return x, s0, dO, dS, euler


def _check(efla, x, S0, dO, dSL, euler):
    c = lambda t: None if t is None else t.cuda()
    got = efla.prefill_bwd(c(x["q"]), c(x["k"]), c(x["v"]), c(x["beta"]), c(S0), c(dO), c(dSL),
                           mode="euler" if euler else "exact")
    torch.cuda.synchronize()
    assert efla.last_error() == 0
    ref = oracle.backward(x["q"], x["k"], x["v"], x["beta"], S0, dO, dSL, euler=euler)
    for name, g, r in zip(("dq", "dk", "dv", "dbeta", "dS0"), got, ref):
        assert_close(g, r, "f32", name)


def test_tiny_fp32(efla):
    _check(efla, *_case("tiny_d32", 1, 2, 256))


def test_tiny_fp32_euler(efla):
    _check(efla, *_case("tiny_d32", 1, 2, 100, euler=True, kscale=32 ** -0.5))


@pytest.mark.parametrize("L", [1, 65, 333])
def test_lm_bf16_inputs(efla, L):
    _check(efla, *_case("lm340m", 2, 3, L))


def test_lm_no_state_no_final_cotangent(efla):
    _check(efla, *_case("lm1p3b", 1, 2, 200, S0=False, dSL=False))


@pytest.mark.parametrize("knorm_idx", [0, 2, 4])
def test_stiffness_fp32(efla, knorm_idx):
    # ||k|| in {1e-3, 1, 100}: the series branch of d alpha / d lambda, the
    # unit range, and saturation alpha ~ 1/lambda
    x = workloads.chunk_inputs("stiffness", B=1, H=2, L=96, knorm=workloads.STIFF_KNORMS[knorm_idx])
    rng = np.random.default_rng(3)
    dO = torch.from_numpy(rng.standard_normal(x["v"].shape).astype(np.float32))
    _check(efla, x, None, dO, None, False)


def test_empty_sequence_passes_dSL_through(efla):
    B, H, d = 1, 2, 64
    z = torch.zeros(B, H, 0, d, device="cuda")
    beta = torch.zeros(B, H, 0, device="cuda")
    dSL = torch.randn(B, H, d, d, device="cuda")
    _, _, _, _, dS0 = efla.prefill_bwd(z, z, z, beta, None, torch.zeros(B, H, 0, d, device="cuda"), dSL)
    torch.cuda.synchronize()
    assert torch.equal(dS0, dSL)
