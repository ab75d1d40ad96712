"""Sequence sharding of one prefill over ranks (the multi-rank half of the
segment-parallel prefill), host logic on CPU with gloo ranks.

Each rank holds one contiguous segment of the sequence.  The helper runs its
segment from zero and from the identity, exchanges the final states with one
all_gather, composes the earlier ranks' affine maps into its true initial
state and reruns.  Here the segment runner is the fp64 oracle and the
composition is plain fp64 arithmetic, so the sharded result must equal the
unsharded oracle to rounding; on GPUs the same helper runs the library's
kernels (efla_chunk_fwd, efla_state_affine) and NCCL."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bounds(L, world):
    # uneven segments on purpose: the later ranks take more tokens
    w = np.arange(1, world + 1, dtype=float)
    b = np.concatenate([[0], np.round(np.cumsum(w) / w.sum() * L)]).astype(int)
    return [(int(b[r]), int(b[r + 1])) for r in range(world)]


def _worker(rank, world, port, L, euler, with_s0, out):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    import workloads
    from delta_rule_linear_03_b200.sequence_parallel import chunk_fwd_sequence_sharded
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        x = workloads.chunk_inputs("tiny_d32", B=1, H=2, L=L)
        if euler:
            x["k"] = x["k"] / 32 ** 0.5  # the explicit step's stable range
        S0 = workloads.random_state(1, 2, 32, seed=7).double() if with_s0 else None
        a, b = _bounds(L, world)[rank]
        seg = {n: x[n][:, :, a:b] for n in ("q", "k", "v", "beta")}

        def segment(q, k, v, beta, S_init, mode, out_dtype):
            o, S = oracle.recurrence(q, k, v, beta, S_init.double(), euler=(mode == "euler"), threads=1)
            return torch.from_numpy(o), torch.from_numpy(S)

        def affine(SI, SZ, X):
            return torch.matmul(SI.double() - SZ.double(), X.double()) + SZ.double()

        o, S = chunk_fwd_sequence_sharded(seg["q"], seg["k"], seg["v"], seg["beta"], S0,
                                          mode="euler" if euler else "exact",
                                          segment=segment, affine=affine)
        ro, rS = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], S0, euler=euler, threads=1)
        err_o = float(np.abs(o.numpy() - ro[:, :, a:b]).max() / np.abs(ro).max())
        err_s = float(np.abs(S.numpy() - rS).max() / np.abs(rS).max()) if rank == world - 1 else 0.0
        out[rank] = (err_o, err_s)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,euler,with_s0", [(2, False, True), (3, False, False), (3, True, True)])
def test_sharded_prefill_equals_unsharded(world, euler, with_s0):
    L = 257  # ragged on every rank
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, L, euler, with_s0, out), nprocs=world, join=True,
                       start_method="spawn")
    assert set(out.keys()) == set(range(world))
    for r in range(world):
        err_o, err_s = out[r]
        assert err_o < 1e-10, f"rank {r}: outputs differ from the unsharded recurrence ({err_o:.2e})"
        assert err_s < 1e-10, f"rank {r}: final state differs ({err_s:.2e})"


def test_initial_state_composition_order():
    # three segments with known affine maps: S_in(2) = M1 (S_end0) + Z1
    from delta_rule_linear_03_b200.sequence_parallel import initial_state
    g = torch.Generator().manual_seed(0)
    S0 = torch.randn(1, 1, 3, 3, generator=g, dtype=torch.float64)
    end0 = torch.randn(1, 1, 3, 3, generator=g, dtype=torch.float64)
    M1 = torch.randn(1, 1, 3, 3, generator=g, dtype=torch.float64)
    Z1 = torch.randn(1, 1, 3, 3, generator=g, dtype=torch.float64)
    maps = [(end0, end0), (Z1, M1 + Z1)]
    aff = lambda SI, SZ, X: torch.matmul(SI - SZ, X) + SZ
    assert torch.equal(initial_state(maps, S0, 0, aff), S0)
    assert torch.equal(initial_state(maps, S0, 1, aff), end0)
    assert torch.allclose(initial_state(maps, S0, 2, aff), torch.matmul(M1, end0) + Z1)
