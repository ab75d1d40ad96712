"""efla_chunk_fwd_noalloc: the prefill entry point for callers that cannot
allocate device memory.

Engines that budget all GPU memory through their own pool, or loops that
cannot afford cudaMalloc's implicit synchronisation, cannot hand the library
a scratch buffer.  This entry point keeps its scratch in a fixed 32 MiB array
inside the library instead.  The tests call it through the C ABI (ctypes) and
hold its results to the results of the regular entry point, efla_chunk_fwd,
on the same inputs, for two calls in a row (the second call finds the first
call's data still in the shared scratch).  This file is collected last so a
failure here never hides the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from parity import BF16_RMS, F32_REL, np64

F32, BF16 = 0, 1


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


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


def _call_noalloc(so, x, S0, o, SL, dtype):
    B, H, L, d = x["q"].shape
    return so.efla_chunk_fwd_noalloc(_p(x["q"]), _p(x["k"]), _p(x["v"]), dtype, 0, _p(x["beta"]), _p(S0), _p(o),
                                     F32, _p(SL), B, H, L, d, d,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _call_regular(so, x, S0, o, SL, dtype):
    B, H, L, d = x["q"].shape
    need = so.efla_chunk_fwd_workspace_size(dtype, B, H, L, d, d)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    return so.efla_chunk_fwd(_p(x["q"]), _p(x["k"]), _p(x["v"]), dtype, 0, _p(x["beta"]), _p(S0), _p(o), F32,
                             _p(SL), B, H, L, d, d, _p(ws) if need else None, need,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(x, ref, dtype):
    x, ref = np64(x), np64(ref)
    if dtype == F32:
        return np.abs(x - ref).max() <= F32_REL * np.abs(ref).max()
    return np.abs(x - ref).max() <= BF16_RMS * np.sqrt(np.mean(ref ** 2))


@pytest.mark.gpu
def test_noalloc_matches_regular_entry_point_twice():
    import delta_rule_linear_03_b200 as efla
    so = efla._lib
    cases = [
        # fp32 tiny workload with a random initial state: both entry points run the CUDA-core kernels
        (workloads.chunk_inputs("tiny_d32"), workloads.random_state(1, 2, 32, seed=11), F32),
        # bf16 at d = 128, shorter: the regular entry point takes the tensor-core kernel here
        (workloads.chunk_inputs("lm340m", B=1, H=3, L=300), None, BF16),
    ]
    for x, S0, dt in cases:
        x = {k: v.cuda() for k, v in x.items() if v is not None}
        S0 = None if S0 is None else S0.cuda()
        B, H, L, d = x["q"].shape
        o_a = torch.empty(B, H, L, d, device="cuda")
        o_b = torch.empty_like(o_a)
        S_a = torch.empty(B, H, d, d, device="cuda")
        S_b = torch.empty_like(S_a)
        assert _call_noalloc(so, x, S0, o_a, S_a, dt) == 0
        assert _call_regular(so, x, S0, o_b, S_b, dt) == 0
        torch.cuda.synchronize()
        assert efla.last_error() == 0
        assert _close(o_a, o_b, dt), "o differs from efla_chunk_fwd"
        assert _close(S_a, S_b, dt), "S_L differs from efla_chunk_fwd"
