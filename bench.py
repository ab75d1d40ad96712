#!/usr/bin/env python
"""Benchmark of the EFLA token mixer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one ``efla_chunk_fwd`` over the lm340m workload (B=8, H=8,
L=2048, d=128, bf16 q/k/v, fp32 beta and state, S0 = 0): gate, UT
transform, state propagation and intra-chunk output all run inside it.
The headline ``value`` is chunked-forward tokens/s (B*L per step; a token
carries all H heads) over all ranks, timed on the device with CUDA events.
The decode metric (batch 64 x 16 heads x d=128, fp32 states) is reported in
the ``decode`` object of the same line.

Inputs are synthetic and seeded (``workloads``); between timed iterations
the step rotates over 3 input/output sets (~410 MB, larger than the 126 MB
L2) so every step reads cold inputs.  Multi-GPU (torchrun, one rank per GPU)
is weak scaling: every rank runs its own independent (b,h) problems with no
collective on the data path; time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle (test infrastructure) on the
host cores on a bounded sample of the same workload and prints the same
line with ``"impl": "reference"``.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

WORKLOAD = "lm340m"
METRIC = "EFLA chunked-fwd tokens/s (% of tensor/HBM roofline); decode tokens/s"
ROTATE = 3


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        j = json.load(open(p))
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                    sm_max_mhz=float(j.get("sm_max_mhz", 1965.0)), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, sm_max_mhz=1965.0, source="fallback")


def ffma_peak_tflops(dev, sm_max_mhz):
    """FP32 FFMA peak derived from unit counts: SMs x 128 fp32 lanes x 2 flop
    (one fused multiply-add) x the maximum SM clock."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return sms * 128 * 2 * sm_max_mhz * 1e6 / 1e12


# ------------------------------------------------------------------ algorithmic work
# DRAM bytes (read + write) of one lm340m efla_chunk_fwd call, summed over its
# two launches, from one ncu capture of the current kernels
# (dram__bytes_read.sum + dram__bytes_write.sum, two calls averaged; prep
# 101.24 + 61.66 MB, serial state kernel 184.60 + 40.95 MB).  Well above the
# 172.5 MB of algorithmic bytes: the prep kernel's per-chunk workspace image
# (-W, M, U) is written and read back once.
CHUNK_TRAFFIC_LM340M = 388.45e6


def chunk_bytes(B, H, L, d, esize, esize_o, s0: bool, sl: bool = True):
    """Algorithmic HBM bytes of one efla_chunk_fwd: read q, k, v and beta,
    write o, read S0 (if given) and write S_L once."""
    tok = B * H * L
    state = B * H * d * d * 4
    return tok * (3 * d * esize + 4 + d * esize_o) + (state if s0 else 0) + (state if sl else 0)


def chunk_flops(B, H, L, d, C=64):
    """Algorithmic flops of the chunked evaluation per head-token:
    6 d^2 (W S, K^T D, Q S) + 5 C d (K K^T, Q K^T, W, U, tril(QK^T) D at
    half density) + C^2/3 (T by forward substitution)."""
    return B * H * L * (6 * d * d + 5 * C * d + C * C / 3.0)


def decode_bytes(B, H, d, esize, esize_o):
    """Read and write the fp32 state once, read q, k, v and beta, write o."""
    return B * H * (2 * 4 * d * d + 3 * d * esize + 4 + d * esize_o)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Reads SM clock and clock-event reasons through NVML (read-only) every
    few milliseconds in a background thread; keeps the samples taken while
    ``active`` is set."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
               0x1: "gpu_idle", 0x10: "sync_boost"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.active = threading.Event()
        self.stop_ = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: the line says so
            self.err = repr(e)
        self.period = period_s
        self.th = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_.is_set():
            if self.active.is_set():
                try:
                    self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                    r = get_r(self.h)
                    for bit, name in self.REASONS.items():
                        if r & bit and name != "gpu_idle":
                            self.reasons.add(name)
                except Exception:
                    pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.th.start()
        return self

    def __exit__(self, *a):
        self.stop_.set()
        if self.ok:
            self.th.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if world != n_gpus and rank == 0:
        print(f"note: --gpus {n_gpus} but WORLD_SIZE {world}", file=sys.stderr)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Max of a per-rank scalar over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w, rank: int) -> int:
    """Each rank draws its own independent (b,h) problems."""
    return 42 + w.index + 1000 * rank


def job_tokens_per_s(world: int, B: int, L: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processed B*L tokens per step; time is
    the slowest rank's."""
    return world * B * L * steps / (ms_max / 1e3)


# ------------------------------------------------------------------ CPU oracle timing
def oracle_rate(x, sample_tokens: int, min_seconds: float, threads: int):
    """tokens/s of the fp64 oracle on the first ``sample_tokens`` tokens of
    every (b,h) of ``x`` (a token = one position of one batch row, all heads)."""
    import oracle
    B, H = x["q"].shape[:2]
    sl = lambda t: t[:, :, :sample_tokens].contiguous()
    q, k, v, beta = (sl(x[n]) for n in ("q", "k", "v", "beta"))
    oracle.recurrence(q[:1, :1, :8], k[:1, :1, :8], v[:1, :1, :8], beta[:1, :1, :8], threads=1)  # load
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.recurrence(q, k, v, beta, None, threads=threads)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds or reps >= 50:
            break
    return B * sample_tokens * reps / dt, dt, reps


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    w = workloads.WORKLOADS[WORKLOAD]
    x = workloads.chunk_inputs(w)
    threads = oracle.default_threads()
    sample = 64  # one chunk-length of tokens of every (b,h) per step
    q, k, v, beta = (x[n][:, :, :sample].contiguous() for n in ("q", "k", "v", "beta"))
    for _ in range(args.warmup):
        oracle.recurrence(q, k, v, beta, None, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.recurrence(q, k, v, beta, None, threads=threads)
    dt = time.perf_counter() - t0
    value = w.B * sample * args.steps / dt
    desc = (f"fp64 sequential oracle, first {sample} tokens of all {w.B}x{w.H} (b,h) of the {WORKLOAD} "
            f"workload per step, {threads} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, workloads.lm340m distribution)",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(w, n):
    return {"workload": f"{w.name}: B={w.B} H={w.H} L={w.L} d={w.d} C=64 {w.dtype} q/k/v, fp32 beta/state/o, S0=0",
            "B": w.B, "H": w.H, "L": w.L, "head_dim": w.d, "chunk": 64, "global_batch": w.B * n,
            "seq_len": w.L, "parallelism": f"dp{n} (independent (b,h) problems per rank, no collective)",
            "l2": f"inputs/outputs rotate over {ROTATE} sets (> L2) between timed steps"}


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import delta_rule_linear_03_b200 as efla

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    w = workloads.WORKLOADS[WORKLOAD]
    B, H, L, d = w.B, w.H, w.L, w.d
    x = workloads.chunk_inputs(w, seed=rank_seed(w, rank))
    sets = []
    for _ in range(ROTATE):
        s = {n: x[n].to(dev) for n in ("q", "k", "v", "beta")}
        s["o"] = torch.empty(B, H, L, d, dtype=torch.float32, device=dev)
        s["S"] = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
        sets.append(s)
    need = efla.workspace_size(x["q"].dtype, B, H, L, d, d)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    launches_per_step = 2 if need else 1
    stream = torch.cuda.current_stream(dev)

    def step(i):
        s = sets[i % ROTATE]
        efla.chunk_fwd(s["q"], s["k"], s["v"], s["beta"], None, o=s["o"], S_L=s["S"], workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    # capture one CUDA graph per input set so Python launch overhead stays off the clock
    graphs = []
    for r in range(ROTATE):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(r)
        graphs.append(g)
    for i in range(max(args.warmup, 3)):
        graphs[i % ROTATE].replay()
    torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        barrier(world)
        torch.cuda.synchronize()
        clk.active.set()
        e0.record(stream)
        for i in range(args.steps):
            graphs[i % ROTATE].replay()
        e1.record(stream)
        torch.cuda.synchronize()
        clk.active.clear()
        barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world)
    ms_step = ms_max / args.steps
    value = job_tokens_per_s(world, B, L, args.steps, ms_max)
    del graphs

    # roofline of the dominant kernel (the whole efla_chunk_fwd when it is one launch)
    nbytes = chunk_bytes(B, H, L, d, 2, 4, s0=False)
    flops = chunk_flops(B, H, L, d)
    achieved_gbs = nbytes / (ms_step / 1e3) / 1e9
    achieved_tf = flops / (ms_step / 1e3) / 1e12

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, workloads.lm340m distribution)",
        "config": workload_config(w, world),
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": achieved_gbs / peaks["hbm"],
                     "traffic": CHUNK_TRAFFIC_LM340M if (WORKLOAD == "lm340m" and launches_per_step == 2) else None,
                     "kernel": "efla_chunk_fwd (all launches of one call)" if launches_per_step > 1
                     else "efla_chunk_fwd fused kernel",
                     "algorithmic_bytes": nbytes, "peak_source": peaks["source"]},
        "roofline_tensor": {"achieved": achieved_tf, "peak": peaks["bf16"], "unit": "TFLOP/s",
                            "frac": achieved_tf / peaks["bf16"], "algorithmic_flops": flops,
                            "peak_source": peaks["source"]},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }

    if rank == 0 and not args.no_decode:
        line["decode"] = bench_decode(efla, dev, args, peaks)
    if rank == 0 and not args.no_longctx:
        line["longctx_prefill"] = bench_longctx(efla, dev, peaks)
    if rank == 0 and not args.no_backward:
        line["backward"] = bench_backward(efla, dev, x, peaks)
    if rank == 0:
        line["gate"] = bench_gate(efla, dev, peaks)
    if rank == 0 and not args.no_stiffness:
        line["stiffness_fp32"] = bench_stiffness(efla, dev, peaks)
    if not args.no_e2e:
        line["e2e"] = bench_e2e(efla, dev, x, args, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        th = oracle.default_threads()
        rate, dt, reps = oracle_rate(x, sample_tokens=L, min_seconds=10.0, threads=th)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": th, "kind": "oracle",
                                "sample": f"full {WORKLOAD} workload x{reps} ({dt:.1f} s), fp64 sequential "
                                          f"recurrence, OpenMP over (b,h)"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def bench_gate(efla, dev, peaks, reps=50):
    """efla_gate alone on the lm1p3b keys (4 x 16 x 4096 bf16 rows of 128;
    67 MB of k, > L2 with 4 rotating copies): alpha and lambda per key.
    CUDA graph of 4 calls over the 4 copies, timed with CUDA events."""
    sets = []
    for i in range(4):
        xi = workloads.chunk_inputs("lm1p3b", seed=100 + i)
        sets.append((xi["k"].to(dev), xi["beta"].to(dev)))
    B, H, L, d = sets[0][0].shape
    outs = [(torch.empty(B, H, L, device=dev), torch.empty(B, H, L, device=dev)) for _ in range(4)]

    def block():
        for (k, b), (a, lam) in zip(sets, outs):
            efla.gate(k, b, alpha=a, lam=lam)

    for _ in range(3):
        block()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        block()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (4 * reps)
    rows = B * H * L
    nbytes = rows * (2 * d + 4 + 8)  # read k (bf16) and beta, write alpha and lambda
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"value": rows / (ms / 1e3), "unit": "keys/s", "ms_per_call": ms, "calls": 4 * reps,
            "config": f"lm1p3b keys: {B}x{H}x{L} rows of d={d} bf16, 4 rotating copies (> L2)",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm"], "traffic": None, "kernel": "gate_kernel",
                         "algorithmic_bytes": nbytes, "peak_source": peaks["source"]}}


def bench_backward(efla, dev, x, peaks, calls=5):
    """efla_prefill_bwd on the timed workload (one fp32 dO, no S0/dS_L):
    exact fp32, one CTA per (b, h) walking the sequence three times."""
    q, k, v, beta = (x[n].to(dev) for n in ("q", "k", "v", "beta"))
    B, H, L, d = k.shape
    dO = torch.randn(B, H, L, d, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
    ws = torch.empty(efla.prefill_bwd_workspace_size(B, H, L, d), dtype=torch.uint8, device=dev)
    for _ in range(2):
        efla.prefill_bwd(q, k, v, beta, None, dO, workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(calls):
        efla.prefill_bwd(q, k, v, beta, None, dO, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    if efla.last_error() != 0:
        raise RuntimeError("efla_prefill_bwd reported a device-side error")
    ms = e0.elapsed_time(e1) / calls
    # HBM bytes: read q, k, v, beta, dO (x2 passes for k); write dq, dk, dv, dbeta; e_t round trip
    tok = B * H * L
    nbytes = tok * (3 * d * 2 + 4 + d * 4 + 3 * d * 4 + 4 + 2 * d * 4)
    return {"value": B * L / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms, "calls": calls,
            "config": f"{WORKLOAD} backward: dq, dk, dv, dbeta, dS0 (fp32), bf16 q/k/v, fp32 dO",
            "kernel": "backward_kernel (fp32, serial over tokens per (b, h))",
            "hbm_bytes_estimate": nbytes}


def bench_longctx(efla, dev, peaks, calls=10):
    """The long-context prefill (B=1, H=16, L=65536, bf16 q/k/v, fp32 o and
    state): 16 heads leave most SMs idle, so the library runs it
    segment-parallel.  Same input twice (1.1 GB of inputs and outputs,
    > L2), CUDA events over `calls` calls after 3 warm-up calls."""
    x = workloads.chunk_inputs("longctx")
    q, k, v, beta = (x[n].to(dev) for n in ("q", "k", "v", "beta"))
    B, H, L, d = k.shape
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=dev)
    S = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    ws = torch.empty(efla.workspace_size(q.dtype, B, H, L, d, d), dtype=torch.uint8, device=dev)
    call = lambda: efla.chunk_fwd(q, k, v, beta, None, o=o, S_L=S, workspace=ws)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(calls):
        call()
    e1.record()
    torch.cuda.synchronize()
    if efla.last_error() != 0:
        raise RuntimeError("efla_chunk_fwd reported a device-side error")
    ms = e0.elapsed_time(e1) / calls
    nbytes = chunk_bytes(B, H, L, d, 2, 4, s0=False)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"value": B * L / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms, "calls": calls,
            "config": f"longctx prefill: B={B} H={H} L={L} d={d} C=64 bf16 q/k/v, fp32 o/state, S0=0",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm"], "traffic": None, "kernel": "efla_chunk_fwd (all launches)",
                         "algorithmic_bytes": nbytes, "peak_source": peaks["source"]}}


def bench_stiffness(efla, dev, peaks, calls=5):
    """The stiffness sweep on the exact-fp32 path: B=2, H=16, L=8192, d=128,
    fp32 q/k/v, ||k|| fixed per run at each of 1e-3, 0.1, 1, 10, 100.  One
    draw: the keys of each run are the unit keys times ||k||, the same fp32
    values the workload generator gives for that norm.  Inputs and outputs
    (0.5 GB) exceed L2; CUDA events over `calls` calls per norm after 2
    warm-up calls.  The path is bound by fp32 arithmetic, so the roofline is
    the FFMA peak."""
    x = workloads.chunk_inputs("stiffness", knorm=1.0)
    q, k1, v, beta = (x[n].to(dev) for n in ("q", "k", "v", "beta"))
    B, H, L, d = k1.shape
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=dev)
    S = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    ws = torch.empty(efla.workspace_size(q.dtype, B, H, L, d, d), dtype=torch.uint8, device=dev)
    per = {}
    for kn in workloads.STIFF_KNORMS:
        k = k1 * kn
        call = lambda: efla.chunk_fwd(q, k, v, beta, None, o=o, S_L=S, workspace=ws)
        for _ in range(2):
            call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(calls):
            call()
        e1.record()
        torch.cuda.synchronize()
        per[kn] = e0.elapsed_time(e1) / calls
        del k
    if efla.last_error() != 0:
        raise RuntimeError("efla_chunk_fwd reported a device-side error")
    ms = statistics.mean(per.values())
    flops = chunk_flops(B, H, L, d)
    tf = flops / (ms / 1e3) / 1e12
    peak = ffma_peak_tflops(dev, peaks["sm_max_mhz"])
    return {"value": B * L / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms,
            "ms_per_knorm": {str(kn): t for kn, t in per.items()}, "calls": calls,
            "config": f"stiffness sweep: B={B} H={H} L={L} d={d} C=64 fp32 q/k/v/o/state, "
                      f"||k|| in {list(workloads.STIFF_KNORMS)}, beta ~ U(0,1), S0=0",
            "roofline": {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "traffic": None, "kernel": "efla_chunk_fwd fp32 path (all launches)",
                         "algorithmic_flops": flops,
                         "peak_source": "derived: SMs x 128 fp32 lanes x 2 flop x max SM clock"},
            "hbm_algorithmic_bytes": chunk_bytes(B, H, L, d, 4, 4, s0=False)}


def bench_decode(efla, dev, args, peaks):
    """Decode: batch 64 x 16 heads x d=128 fp32 states, bf16 q/k/v, one
    token per step.  Steps rotate over 4 state sets (256 MB > L2) and are
    replayed from a CUDA graph of 8 steps."""
    Bd, Hd, d = workloads.DECODE_BATCH, workloads.DECODE_HEADS, 128
    nsets = 4
    xin = workloads.decode_inputs(8)
    ins = [{n: xin[n][i].to(dev) for n in ("q", "k", "v", "beta")} for i in range(8)]
    states = [workloads.random_state(Bd, Hd, d, seed=s).to(dev) for s in range(nsets)]
    outs = [torch.empty(Bd, Hd, d, dtype=torch.float32, device=dev) for _ in range(8)]

    def block():
        for i in range(8):
            efla.decode_step(ins[i]["q"], ins[i]["k"], ins[i]["v"], ins[i]["beta"], states[i % nsets], o=outs[i])

    for _ in range(3):
        block()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        block()
    reps = max(1, args.steps // 8)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms_step = e0.elapsed_time(e1) / (8 * reps)
    nbytes = decode_bytes(Bd, Hd, d, 2, 4)
    gbs = nbytes / (ms_step / 1e3) / 1e9
    return {"value": Bd / (ms_step / 1e3), "unit": "tokens/s", "ms_per_step": ms_step, "steps": 8 * reps,
            "config": f"batch {Bd} x {Hd} heads x d={d}, fp32 states, bf16 q/k/v, fp32 o, {nsets} state sets (> L2)",
            "gpu_launches": 8 * reps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm"], "traffic": None, "kernel": "decode_kernel",
                         "algorithmic_bytes": nbytes, "peak_source": peaks["source"]}}


def bench_e2e(efla, dev, x, args, world):
    """The same metric through the public API from pinned host buffers:
    every step copies q, k, v, beta host->device, runs efla_chunk_fwd and
    copies o and S_L device->host."""
    hq, hk, hv, hb = (x[n].pin_memory() for n in ("q", "k", "v", "beta"))
    B, H, L, d = hq.shape
    ho = torch.empty(B, H, L, d, dtype=torch.float32).pin_memory()
    hS = torch.empty(B, H, d, d, dtype=torch.float32).pin_memory()
    dq, dk, dv, db = (torch.empty_like(t, device=dev) for t in (hq, hk, hv, hb))
    do = torch.empty(B, H, L, d, dtype=torch.float32, device=dev)
    dS = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)

    def step():
        for dst, src in ((dq, hq), (dk, hk), (dv, hv), (db, hb)):
            dst.copy_(src, non_blocking=True)
        efla.chunk_fwd(dq, dk, dv, db, None, o=do, S_L=dS)
        ho.copy_(do, non_blocking=True)
        hS.copy_(dS, non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 30))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record()
    for _ in range(n):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hb))
    d2h = ho.numel() * ho.element_size() + hS.numel() * hS.element_size()
    return {"value": world * B * L * n / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-longctx", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-stiffness", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
