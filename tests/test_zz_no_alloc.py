"""efla_chunk_fwd_noalloc: the prefill entry point for callers that cannot
allocate device memory.

Engines that budget all GPU memory through their own pool, or loops that
cannot afford cudaMalloc's implicit synchronisation, cannot hand the library
a scratch buffer.  This entry point keeps its scratch in a fixed 32 MiB array
inside the library instead.  The tests call it through the C ABI (ctypes) and
check it
* against the fp64 oracle on the tiny fp32 workload and on a bf16 case;
* against the regular entry point, efla_chunk_fwd, on a case that fills
  nearly the whole array (400 head-chunks of 64 tokens at d = 128; the
  regular entry point runs the tensor-core kernels there, a different path);
* for an in-place state update (S_L = S0);
* for two calls in a row on the same inputs, whose results must be
  bit-identical (the second call finds the first call's data still in the
  shared array and must not depend on it).
This file is collected last so a failure here never hides the other tests.
"""
import ctypes

import pytest
import torch

import oracle
import workloads
from parity import assert_close

F32, BF16 = 0, 1


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_noalloc_rejects_oversize_before_launch():
    """Sizes whose scratch exceeds the fixed array are refused up front
    (EFLA_ERR_WORKSPACE), without any CUDA call; runs on a CPU-only host."""
    import delta_rule_linear_03_b200 as efla
    so = efla._lib
    cap = efla.NOALLOC_SCRATCH_BYTES
    assert so.efla_chunk_fwd_workspace_size_simt(1, 1, 64, 128, 128) * 409 <= cap
    assert so.efla_chunk_fwd_workspace_size_simt(1, 1, 64, 128, 128) * 410 > cap
    A = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(6)]
    # 410 chunks of 64 tokens at d = 128 do not fit
    st = so.efla_chunk_fwd_noalloc(A[0], A[1], A[2], BF16, 0, A[3], None, A[4], F32, A[5], 1, 1, 410 * 64,
                                   128, 128, None)
    assert st == 8  # EFLA_ERR_WORKSPACE
    st = so.efla_chunk_fwd_noalloc(A[0], A[1], A[2], F32, 0, A[3], None, A[4], F32, None, 2, 3, 64, 48, 48, None)
    assert st == 5  # unsupported head size, as in efla_chunk_fwd


def _noalloc(so, x, S0, o, SL, dtype):
    B, H, L, d = x["q"].shape
    return so.efla_chunk_fwd_noalloc(_p(x["q"]), _p(x["k"]), _p(x["v"]), dtype, 0, _p(x["beta"]), _p(S0), _p(o),
                                     F32, _p(SL), B, H, L, d, d, _stream())


def _regular(so, x, S0, o, SL, dtype):
    B, H, L, d = x["q"].shape
    need = so.efla_chunk_fwd_workspace_size(dtype, B, H, L, d, d)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    return so.efla_chunk_fwd(_p(x["q"]), _p(x["k"]), _p(x["v"]), dtype, 0, _p(x["beta"]), _p(S0), _p(o), F32,
                             _p(SL), B, H, L, d, d, _p(ws) if need else None, need, _stream())


def _outputs(x):
    B, H, L, d = x["q"].shape
    return torch.empty(B, H, L, d, device="cuda"), torch.empty(B, H, d, d, device="cuda")


def _gpu(x):
    return {k: v.cuda() for k, v in x.items() if v is not None}


CASES = [
    # fp32 tiny workload with a random initial state
    ("tiny_d32", dict(), workloads.random_state(1, 2, 32, seed=11), F32, "f32"),
    # bf16 at d = 128
    ("lm340m", dict(B=1, H=3, L=300), None, BF16, "bf16"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw,S0,dt,tag", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_oracle_twice(name, kw, S0, dt, tag):
    """Two calls in a row on the same inputs: each meets the parity bar
    against the fp64 oracle, and the two results are bit-identical."""
    import delta_rule_linear_03_b200 as efla
    so = efla._lib
    xc = workloads.chunk_inputs(name, **kw)
    x = _gpu(xc)
    S0g = None if S0 is None else S0.cuda()
    (o1, S1), (o2, S2) = _outputs(x), _outputs(x)
    assert _noalloc(so, x, S0g, o1, S1, dt) == 0
    assert _noalloc(so, x, S0g, o2, S2, dt) == 0
    torch.cuda.synchronize()
    assert efla.last_error() == 0
    ro, rS = oracle.recurrence(xc["q"], xc["k"], xc["v"], xc["beta"], S0)
    assert_close(o1, ro, tag, "o")
    assert_close(S1, rS, tag, "S_L")
    assert torch.equal(o1, o2) and torch.equal(S1, S2), "second call differs from the first"


@pytest.mark.gpu
def test_noalloc_in_place_state():
    import delta_rule_linear_03_b200 as efla
    so = efla._lib
    xc = workloads.chunk_inputs("lm1p3b", B=1, H=2, L=200)
    x = _gpu(xc)
    S = xc["S0"].cuda()
    o = torch.empty(1, 2, 200, 128, device="cuda")
    assert _noalloc(so, x, S, o, S, BF16) == 0
    torch.cuda.synchronize()
    assert efla.last_error() == 0
    ro, rS = oracle.recurrence(xc["q"], xc["k"], xc["v"], xc["beta"], xc["S0"])
    assert_close(o, ro, "bf16", "o")
    assert_close(S, rS, "bf16", "S_L")


@pytest.mark.gpu
def test_noalloc_near_full_array_matches_regular_entry_point():
    """400 head-chunks at d = 128 use 32.8 of the 33.6 MB of the array; the
    regular entry point (tensor-core kernels) gives the same result within
    the bf16 bar, and both meet it against the oracle on sampled heads."""
    import delta_rule_linear_03_b200 as efla
    so = efla._lib
    B, H, L = 1, 4, 100 * 64
    assert so.efla_chunk_fwd_workspace_size_simt(B, H, L, 128, 128) > 0.97 * efla.NOALLOC_SCRATCH_BYTES
    xc = workloads.chunk_inputs("lm1p3b", B=B, H=H, L=L)
    x = _gpu(xc)
    S0 = xc["S0"].cuda()
    (o_a, S_a), (o_b, S_b) = _outputs(x), _outputs(x)
    assert _noalloc(so, x, S0, o_a, S_a, BF16) == 0
    assert _regular(so, x, S0, o_b, S_b, BF16) == 0
    torch.cuda.synchronize()
    assert efla.last_error() == 0
    assert_close(o_a, o_b, "bf16", "o vs efla_chunk_fwd")
    assert_close(S_a, S_b, "bf16", "S_L vs efla_chunk_fwd")
    for h in (0, 3):
        sl = lambda t: t[:, h:h + 1]
        ro, rS = oracle.recurrence(sl(xc["q"]), sl(xc["k"]), sl(xc["v"]), sl(xc["beta"]), sl(xc["S0"]))
        assert_close(o_a[:, h:h + 1], ro, "bf16", f"o[{h}]")
        assert_close(S_a[:, h:h + 1], rS, "bf16", f"S_L[{h}]")
