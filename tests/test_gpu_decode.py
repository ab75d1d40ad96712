"""efla_decode_step on the GPU against the oracle recurrence at L = 1."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import assert_close, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def efla():
    import delta_rule_linear_03_b200 as m
    return m


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("mode", ["exact", "euler"])
def test_decode_steps_long_context_batch(efla, dtype, mode):
    """Batch 64 x 16 heads x d=128 (the long-context decode shape), several
    chained steps from a random state."""
    steps = 4
    x = workloads.decode_inputs(steps, dtype=dtype)
    S = workloads.random_state(workloads.DECODE_BATCH, workloads.DECODE_HEADS, 128)
    Sg = S.cuda()
    Sref = np64(S)
    for s in range(steps):
        o = efla.decode_step(x["q"][s].cuda(), x["k"][s].cuda(), x["v"][s].cuda(), x["beta"][s].cuda(), Sg,
                             mode=mode, out_dtype=torch.bfloat16 if s % 2 else torch.float32)
        ro, Sref = oracle.decode_step(x["q"][s], x["k"][s], x["v"][s], x["beta"][s], Sref,
                                      euler=(mode == "euler"))
        assert_close(o, ro, dtype, f"o step {s}", out_bf16=bool(s % 2))
    torch.cuda.synchronize()
    # the state is fp32 in both arms: hold it to the fp32 bar
    assert_close(Sg, Sref, "f32", "S")


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_head_sizes(efla, d, dtype):
    g = torch.Generator().manual_seed(100 + d)
    B, H = 3, 5
    q = torch.randn(B, H, d, generator=g).to(dtype)
    k = (torch.randn(B, H, d, generator=g) * 0.3).to(dtype)
    v = torch.randn(B, H, d, generator=g).to(dtype)
    beta = torch.rand(B, H, generator=g)
    S = torch.randn(B, H, d, d, generator=g)
    Sg = S.cuda()
    o = efla.decode_step(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), Sg)
    ro, rS = oracle.decode_step(q, k, v, beta, S)
    tag = "f32" if dtype == torch.float32 else "bf16"
    assert_close(o, ro, tag, "o")
    assert_close(Sg, rS, "f32", "S")


def test_decode_equals_prefill_chain(efla):
    """L decode steps from S0 reproduce the tiny workload's full recurrence."""
    x = workloads.chunk_inputs("tiny_d32", L=40)
    S = torch.zeros(1, 2, 32, 32, device="cuda")
    outs = []
    for t in range(40):
        outs.append(efla.decode_step(x["q"][:, :, t].cuda(), x["k"][:, :, t].cuda(), x["v"][:, :, t].cuda(),
                                     x["beta"][:, :, t].cuda(), S))
    o = torch.stack(outs, dim=2)
    ro, rS = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"])
    assert_close(o, ro, "f32", "o")
    assert_close(S, rS, "f32", "S")


def test_decode_zero_key_and_zero_beta(efla):
    d = 64
    q = torch.randn(1, 2, d)
    k = torch.zeros(1, 2, d)
    k[0, 1] = torch.randn(d)
    v = torch.randn(1, 2, d)
    beta = torch.tensor([[0.5, 0.0]])
    S = torch.randn(1, 2, d, d)
    Sg = S.cuda()
    o = efla.decode_step(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), Sg)
    ro, rS = oracle.decode_step(q, k, v, beta, S)
    # k = 0 and beta = 0 both leave the state unchanged
    np.testing.assert_array_equal(np64(Sg), np64(S))
    assert_close(o, ro, "f32", "o")
