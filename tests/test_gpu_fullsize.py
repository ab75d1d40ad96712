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
    """L = 65536 prefill (two sampled heads), then the full long-context
    decode: 1024 chained efla_decode_step calls at batch 64 x 16 heads,
    every state starting as a copy of the prefill state of its head.

    The oracle follows a sample of (b, h) states through all 1024 steps:
    * from the GPU's prefill state, so the comparison isolates the decode
      chain (o at the bf16 bar on a sample of steps; the fp32 state after
      the last step at the fp32 bar);
    * from the oracle's own prefill state, for the end-to-end chain
      (prefill then decode) at the bf16 bar."""
    x = workloads.chunk_inputs("longctx")
    q, k, v, beta = (x[n].cuda() for n in ("q", "k", "v", "beta"))
    o, SL = efla.chunk_fwd(q, k, v, beta, None)
    torch.cuda.synchronize()
    assert efla.last_error() == 0
    heads = (0, 11)
    rS_pref = {}
    for h in heads:
        sl = lambda t: t[:, h:h + 1]
        ro, rS = oracle.recurrence(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta"]))
        assert_close(o[:, h:h + 1], ro, "bf16", f"o[{h}]")
        assert_close(SL[:, h:h + 1], rS, "bf16", f"S_L[{h}]")
        rS_pref[h] = rS[0, 0]
    del o, q, k, v, beta

    Bd, Hd, steps = workloads.DECODE_BATCH, workloads.DECODE_HEADS, workloads.DECODE_STEPS
    S = SL.expand(Bd, -1, -1, -1).contiguous()
    SL_host = SL[0].double().cpu().numpy()
    # (b, h) pairs the oracle follows: decode-only from the GPU prefill state,
    # and end to end from the oracle's prefill state (heads it computed above)
    pairs = [(0, 3), (17, 11), (33, 7), (50, 0), (63, 15)]
    e2e_pairs = [(5, 0), (40, 11), (63, 0)]
    bi = torch.tensor([b for b, _ in pairs]); hi = torch.tensor([h for _, h in pairs])
    be = torch.tensor([b for b, _ in e2e_pairs]); he = torch.tensor([h for _, h in e2e_pairs])
    Sref = SL_host[hi.numpy()][None].copy()                           # [1, P, d, d]
    Se2e = np.stack([rS_pref[h] for _, h in e2e_pairs])[None].copy()  # [1, E, d, d]
    check_at = {0, 1, 2, 255, 511, 767, 1000, steps - 1}
    block = 64
    for s0 in range(0, steps, block):
        d = workloads.decode_inputs(block, first=s0)
        for j in range(block):
            s = s0 + j
            qs, ks, vs, bs = d["q"][j], d["k"][j], d["v"][j], d["beta"][j]
            od = efla.decode_step(qs.cuda(), ks.cuda(), vs.cuda(), bs.cuda(), S)
            pick = lambda t, b, h: t[b, h][None]
            ro, Sref = oracle.decode_step(pick(qs, bi, hi), pick(ks, bi, hi), pick(vs, bi, hi),
                                          pick(bs, bi, hi), Sref)
            re, Se2e = oracle.decode_step(pick(qs, be, he), pick(ks, be, he), pick(vs, be, he),
                                          pick(bs, be, he), Se2e)
            if s in check_at:
                odc = od.cpu()
                assert_close(odc[bi, hi][None], ro, "bf16", f"decode o step {s}")
                assert_close(odc[be, he][None], re, "bf16", f"prefill+decode o step {s}")
    torch.cuda.synchronize()
    assert efla.last_error() == 0
    Sc = S.cpu()
    assert_close(Sc[bi, hi][None], Sref, "f32", f"decode S after {steps} steps")
    assert_close(Sc[be, he][None], Se2e, "bf16", f"prefill+decode S after {steps} steps")
