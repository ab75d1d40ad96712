"""Parity at the full workload sizes, in the launch configuration the
benchmark times.  The oracle recomputes every (b,h) it checks from scratch;
for the largest workloads it checks a sample of heads (each head is an
independent recurrence, so a sampled head is checked exactly)."""
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


def check_heads(efla, x, dtype, heads=None):
    q, k, v, beta = (x[n].cuda() for n in ("q", "k", "v", "beta"))
    S0 = None if x["S0"] is None else x["S0"].cuda()
    o, SL = efla.chunk_fwd(q, k, v, beta, S0)
    torch.cuda.synchronize()
    assert efla.last_error() == 0, "a device-side wait timed out"
    B, H = x["q"].shape[:2]
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in pairs:
        sl = lambda t: None if t is None else t[b:b + 1, h:h + 1]
        ro, rS = oracle.recurrence(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta"]), sl(x["S0"]))
        assert_close(o[b:b + 1, h:h + 1], ro, dtype, f"o[{b},{h}]")
        assert_close(SL[b:b + 1, h:h + 1], rS, dtype, f"S_L[{b},{h}]")


def test_lm340m_full(efla):
    x = workloads.chunk_inputs("lm340m")
    check_heads(efla, x, "bf16", heads=[(b, h) for b in range(8) for h in range(0, 8, 3)])


def test_lm1p3b_full(efla):
    x = workloads.chunk_inputs("lm1p3b")
    check_heads(efla, x, "bf16", heads=[(b, h) for b in range(4) for h in (0, 7, 15)])


@pytest.mark.parametrize("knorm", workloads.STIFF_KNORMS)
def test_stiffness_full(efla, knorm):
    x = workloads.chunk_inputs("stiffness", knorm=knorm)
    check_heads(efla, x, "f32", heads=[(0, 0), (0, 9), (1, 4), (1, 15)])


def test_longctx_prefill_full_then_decode(efla):
    """L = 65536 prefill (two sampled heads), then decode steps at batch 64
    starting from copies of the prefill state."""
    x = workloads.chunk_inputs("longctx")
    q, k, v, beta = (x[n].cuda() for n in ("q", "k", "v", "beta"))
    o, SL = efla.chunk_fwd(q, k, v, beta, None)
    torch.cuda.synchronize()
    for h in (0, 11):
        sl = lambda t: t[:, h:h + 1]
        ro, rS = oracle.recurrence(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta"]))
        assert_close(o[:, h:h + 1], ro, "bf16", f"o[{h}]")
        assert_close(SL[:, h:h + 1], rS, "bf16", f"S_L[{h}]")
    # decode: 64 copies of the prefill state, 3 steps
    S = SL.expand(workloads.DECODE_BATCH, -1, -1, -1).contiguous()
    Sref = S.double().cpu().numpy()
    d = workloads.decode_inputs(3)
    for s in range(3):
        od = efla.decode_step(d["q"][s].cuda(), d["k"][s].cuda(), d["v"][s].cuda(), d["beta"][s].cuda(), S)
        ro, Sref = oracle.decode_step(d["q"][s], d["k"][s], d["v"][s], d["beta"][s], Sref)
        assert_close(od, ro, "bf16", f"decode o step {s}")
    torch.cuda.synchronize()
    assert_close(S, Sref, "f32", "decode S")
