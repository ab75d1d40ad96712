"""efla_gate on the GPU against the oracle's gate (fp64)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def efla():
    import delta_rule_linear_03_b200 as m
    return m


@pytest.mark.parametrize("name,L", [("tiny_d32", 256), ("lm340m", 300), ("lm1p3b", 77)])
@pytest.mark.parametrize("mode", ["exact", "euler"])
def test_gate_matches_oracle(efla, name, L, mode):
    x = workloads.chunk_inputs(name, L=L)
    a, lam = efla.gate(x["k"].cuda(), x["beta"].cuda(), mode=mode)
    ra, rl = oracle.gate(x["k"], x["beta"], euler=(mode == "euler"))
    np.testing.assert_allclose(np64(lam), rl, rtol=2e-6, atol=0)
    np.testing.assert_allclose(np64(a), ra, rtol=2e-6, atol=0)


@pytest.mark.parametrize("knorm", workloads.STIFF_KNORMS)
def test_gate_stiffness_sweep(efla, knorm):
    """||k|| from 1e-3 to 100: expm1 precision at beta*lambda -> 0 and the
    saturation alpha -> 1/lambda at large beta*lambda."""
    x = workloads.chunk_inputs("stiffness", B=1, H=4, L=1000, knorm=knorm)
    a, lam = efla.gate(x["k"].cuda(), x["beta"].cuda())
    ra, rl = oracle.gate(x["k"], x["beta"])
    np.testing.assert_allclose(np64(lam), rl, rtol=2e-6)
    np.testing.assert_allclose(np64(a), ra, rtol=2e-6)


def test_gate_edge_values(efla):
    """k = 0 (lambda = 0 -> alpha = beta), tiny and huge lambda, beta = 0, and
    a ragged row count (not a multiple of the rows one warp covers)."""
    d = 128
    L = 13
    k = torch.zeros(1, 1, L, d)
    k[0, 0, 1, 0] = 1e-7          # lambda = 1e-14 < clamp
    k[0, 0, 2, :] = 1e-3          # lambda = 1.28e-4
    k[0, 0, 3, :] = 30.0          # lambda = 115200, saturated
    k[0, 0, 4:, :] = torch.linspace(-2, 2, d)
    beta = torch.tensor([[[0.5, 0.7, 0.2, 0.9, 0.0, 1.0, 3.0, 0.1, 0.5, 0.5, 0.5, 0.5, 0.5]]])
    a, lam = efla.gate(k.cuda(), beta.cuda())
    ra, rl = oracle.gate(k, beta)
    np.testing.assert_allclose(np64(a), ra, rtol=2e-6)
    np.testing.assert_allclose(np64(lam), rl, rtol=2e-6)
    assert np64(a)[0, 0, 0] == pytest.approx(0.5, rel=1e-7)
    assert np64(a)[0, 0, 4] == 0.0


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gate_head_sizes(efla, d, dtype):
    g = torch.Generator().manual_seed(d)
    k = torch.randn(3, 5, 37, d, generator=g).to(dtype)
    beta = torch.rand(3, 5, 37, generator=g)
    a, lam = efla.gate(k.cuda(), beta.cuda())
    ra, rl = oracle.gate(k, beta)
    np.testing.assert_allclose(np64(a), ra, rtol=2e-6)
    np.testing.assert_allclose(np64(lam), rl, rtol=2e-6)
