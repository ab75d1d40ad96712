"""Segment-parallel bf16 prefill (few heads, long sequences) on the GPU
against the sequential fp64 oracle.

With few (b, h) problems the chunk path splits the sequence into P
segments: pass A runs segment 0 from S0 and every middle segment from zero
and from the identity, a chain of fp32 products composes the segments'
affine state maps, pass B reruns segments 1..P-1 from their true initial
states.  A middle segment's two pass-A runs share one CTA per d_v half
(128 state columns: from zero and from the identity).  The shapes below
select P = 3 (49 chunks) and P = 8 (128 chunks); the full-size long-context
test in test_gpu_fullsize.py runs P = 5."""
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


def run(efla, x, mode="exact", S0=None, out_dtype=torch.float32):
    o, SL = efla.chunk_fwd(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["beta"].cuda(),
                           None if S0 is None else S0.cuda(), mode=mode, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert efla.last_error() == 0, "a device-side wait timed out"
    return o, SL


@pytest.mark.parametrize("L", [3100, 8192])
def test_segmented_with_initial_state(efla, L):
    x = workloads.chunk_inputs("lm1p3b", B=1, H=2, L=L)
    o, SL = run(efla, x, S0=x["S0"])
    ro, rS = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], x["S0"])
    assert_close(o, ro, "bf16", "o")
    assert_close(SL, rS, "bf16", "S_L")


def test_segmented_zero_state_bf16_out(efla):
    x = workloads.chunk_inputs("lm340m", B=1, H=3, L=3333)
    o, SL = run(efla, x, out_dtype=torch.bfloat16)
    ro, rS = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], None)
    assert_close(o, ro, "bf16", "o", out_bf16=True)
    assert_close(SL, rS, "bf16", "S_L")


def test_segmented_euler(efla):
    x = workloads.chunk_inputs("lm340m", B=1, H=2, L=3072)
    # the explicit-Euler step I - beta k k^T is unstable once beta ||k||^2 > 2
    # (section 关键设计 1); scale the keys into its stable range
    x["k"] = (x["k"].float() / 3).to(x["k"].dtype)
    o, SL = run(efla, x, mode="euler")
    ro, rS = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], None, euler=True)
    assert_close(o, ro, "bf16", "o")
    assert_close(SL, rS, "bf16", "S_L")


def test_segmented_in_place_state(efla):
    # S_L written over S0: pass A reads S0 before pass B overwrites it
    x = workloads.chunk_inputs("lm1p3b", B=1, H=2, L=4096)
    S = x["S0"].clone().cuda()
    efla.chunk_fwd(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["beta"].cuda(), S, S_L=S)
    torch.cuda.synchronize()
    assert efla.last_error() == 0
    _, rS = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], x["S0"])
    assert_close(S, rS, "bf16", "S_L in place")


def test_state_affine_matches_fp64(efla):
    g = torch.Generator().manual_seed(3)
    for d in (32, 64, 128):
        SI, SZ, X = (torch.randn(2, 3, d, d, generator=g) for _ in range(3))
        out = efla.state_affine(SI.cuda(), SZ.cuda(), X.cuda())
        torch.cuda.synchronize()
        ref = torch.matmul(SI.double() - SZ.double(), X.double()) + SZ.double()
        err = (out.cpu().double() - ref).abs().max().item() / ref.abs().max().item()
        assert err < 1e-5, f"d={d}: rel err {err:.2e}"


def test_sequence_sharded_helper_on_one_gpu(efla):
    # the rank-by-rank steps of the sequence-sharded helper, run here one
    # segment after another on one GPU with the library's kernels
    from delta_rule_linear_03_b200.sequence_parallel import initial_state
    x = workloads.chunk_inputs("lm1p3b", B=1, H=2, L=700)
    S0 = x["S0"].cuda()
    bounds = [(0, 200), (200, 457), (457, 700)]
    d = 128
    eye = torch.eye(d, device="cuda").expand(1, 2, d, d).contiguous()
    zero = torch.zeros(1, 2, d, d, device="cuda")
    segs = [{n: x[n][:, :, a:b].contiguous().cuda() for n in ("q", "k", "v", "beta")} for a, b in bounds]
    maps = []
    for r, s in enumerate(segs):
        if r == 0:
            _, S_end = efla.chunk_fwd(s["q"], s["k"], s["v"], s["beta"], S0)
            maps.append((S_end, S_end))
        else:
            _, SZ = efla.chunk_fwd(s["q"], s["k"], s["v"], s["beta"], zero)
            _, SI = efla.chunk_fwd(s["q"], s["k"], s["v"], s["beta"], eye)
            maps.append((SZ, SI))
    outs = []
    for r, s in enumerate(segs):
        S_in = initial_state(maps, S0, r, efla.state_affine)
        o, S_last = efla.chunk_fwd(s["q"], s["k"], s["v"], s["beta"], S_in.contiguous())
        outs.append(o)
    torch.cuda.synchronize()
    assert efla.last_error() == 0
    ro, rS = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], x["S0"])
    assert_close(torch.cat(outs, dim=2), ro, "bf16", "o")
    assert_close(S_last, rS, "bf16", "S_L")
