"""The device-side failure path: a bounded wait that runs out reports
EFLA_ERR_TIMEOUT through the sticky error word and leaves the CUDA context
usable.  The wait is on an mbarrier that nothing ever arrives on; nothing
faults, traps or hangs."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import delta_rule_linear_03_b200 as efla
    assert efla.last_error() == 0
    st = torch.cuda.current_stream().cuda_stream
    import ctypes
    assert efla._lib.efla_diag_wait_timeout(2_000_000, ctypes.c_void_p(st)) == 0  # ~1 ms of SM clock
    assert efla.last_error() == 7  # EFLA_ERR_TIMEOUT, and the word is cleared
    assert efla.last_error() == 0
    # the context still runs real work correctly afterwards
    x = workloads.chunk_inputs("tiny_d32", L=70)
    o, SL = efla.chunk_fwd(*(x[n].cuda() for n in ("q", "k", "v", "beta")), None)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and efla.last_error() == 0


def test_diag_rejects_bad_limit():
    import delta_rule_linear_03_b200 as efla
    assert efla._lib.efla_diag_wait_timeout(0, None) == 2
