"""The N > 1 host path of bench.py on CPU: two gloo ranks.

Every (b,h) is an independent recurrence, so ranks share no data; the only
cross-rank steps are the barrier and the max over ranks of the timed
region.  These run here on the gloo backend; on GPUs bench.py runs the same
code on NCCL."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import workloads
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        w = workloads.WORKLOADS["lm340m"]
        # each rank's problems come from its own seed
        x = workloads.chunk_inputs(w, B=1, H=2, L=40, seed=bench.rank_seed(w, rank))
        # per-rank "time": rank-dependent; the job time is the max over ranks
        ms = 10.0 + rank
        bench.barrier(world)
        ms_max = bench.max_over_ranks(ms, world, device="cpu")
        # the per-rank result is an independent oracle evaluation of its own inputs
        o, S = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], threads=1)
        out[rank] = (ms_max, float(x["q"].float().sum()), float(o.sum()),
                     bench.job_tokens_per_s(world, 8, 2048, 100, ms_max))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_independent_shards():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert set(out.keys()) == {0, 1}
    # both ranks agree on the slowest rank's time
    assert out[0][0] == out[1][0] == 11.0
    # the shards differ (independent seeds) and so do their results
    assert out[0][1] != out[1][1] and out[0][2] != out[1][2]
    # whole-job throughput counts every rank's tokens over the max time
    assert out[0][3] == pytest.approx(2 * 8 * 2048 * 100 / 0.011)


def test_reference_arm_non_zero_rank_does_nothing(capsys, monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""
