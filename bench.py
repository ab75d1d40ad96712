#!/usr/bin/env python
"""Benchmark of the EFLA token mixer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one ``efla_chunk_fwd`` over the long-context prefill workload
(B=1, H=16, L=65536, d=128, bf16 q/k/v, fp32 beta, state and o, S0 = 0),
the largest configuration that the metric is quoted on and that fits one
GPU: gate, UT transform, state propagation and intra-chunk output all run
inside it.  The headline ``value`` is chunked-forward tokens/s (B*L per
step; a token carries all H heads) over all ranks, timed on the device with
CUDA events around K replays of a CUDA graph of one call.  Its inputs and
outputs (1.1 GB) are larger than the 126 MB L2, so every step reads them
from HBM.

The same line carries, under ``configs``, every workload of the metric:
``tiny_d32``, ``lm340m``, ``lm1p3b`` (random S0), ``stiffness`` (all five
key norms, exact-fp32 path), the long-context prefill (the headline) and
its 1024-step decode at batch 64 x 16 heads; each with its roofline and a
CPU baseline (the fp64 oracle at 1 thread and at all host threads, on a
bounded sample).  ``deltanet_vs_efla`` times the DeltaNet (explicit Euler)
mode against the exact gate through the same kernels.

Inputs are synthetic and seeded (``workloads``).  Multi-GPU (torchrun, one
rank per GPU) is weak scaling: every rank runs its own independent (b,h)
problems with no collective on the data path; time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle (test infrastructure) on the
host cores on a bounded sample of the same workload and prints the same
line with ``"impl": "reference"``.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import platform
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

WORKLOAD = "longctx"
METRIC = "EFLA chunked-fwd tokens/s (% of tensor/HBM roofline); decode tokens/s"


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


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


# ------------------------------------------------------------------ algorithmic work
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one
# long-context efla_chunk_fwd call, all launches: an ncu capture of the same
# call at L = 16384 (16 heads, the same segmented kernels and plan shape)
# measured 733.3 MB read + 274.0 MB written per call; the per-chunk work and
# images scale with L, so the full call moves about 4 x 1007.3 MB.  It is
# 3.7 x the algorithmic bytes: the per-chunk workspace image (-W, M, U)
# makes a round trip, and pass A and pass B both read the middle segments.
LONGCTX_TRAFFIC = 4 * 1007.3e6


def chunk_bytes(B, H, L, d, esize, esize_o, s0: bool, sl: bool = True):
    """HBM bytes of one efla_chunk_fwd that the method itself needs: read q,
    k, v and beta, write o, read S0 (if given) and write S_L once.  With o in
    the q dtype this is the per-unit figure 3 d e + 4 + d e per head-token
    (1028 B in bf16 at d = 128) plus 64 KB per (b, h) per state read or write."""
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


def chunk_launches(efla, dtype, B, H, L, d):
    """Kernel launches of one efla_chunk_fwd.  The tensor-core path runs the
    prep kernel and one serial launch, or, segment-parallel (when the
    workspace holds segment states past the per-chunk images), four: the
    prep, pass A, the segment chain and pass B.  The CUDA-core path runs two
    kernels."""
    if dtype != torch.bfloat16 or d != 128:
        return 2
    nc = (L + 63) // 64
    image = efla.workspace_size(dtype, 1, 1, 64, d, d)  # one chunk's image (never segmented)
    return 4 if efla.workspace_size(dtype, B, H, L, d, d) > B * H * nc * image else 2


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


# ------------------------------------------------------------------ timing helpers
def graph_of(fn):
    """Capture one call of ``fn`` into a CUDA graph (after it ran eagerly)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_replays(graphs, reps, stream=None):
    """Mean ms per replay of ``reps`` replays cycling over ``graphs``, CUDA
    events on the current stream, synchronised on both sides."""
    stream = stream or torch.cuda.current_stream()
    for i in range(3):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(reps):
        graphs[i % len(graphs)].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def hbm_roofline(nbytes, ms, peaks, kernel, traffic=None, note=None):
    gbs = nbytes / (ms / 1e3) / 1e9
    r = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s", "frac": gbs / peaks["hbm"],
         "traffic": traffic, "kernel": kernel, "algorithmic_bytes": nbytes,
         "peak_source": f"{peaks['source']} (copy bandwidth)"}
    if note:
        r["note"] = note
    return r


# ------------------------------------------------------------------ CPU oracle timing
def oracle_rate(x, heads, sample_tokens: int, threads: int, min_seconds: float):
    """Head-tokens/s of the fp64 oracle on the first ``sample_tokens`` tokens
    of the (b, h) pairs ``heads`` of ``x``; repeats until ``min_seconds``."""
    import oracle
    bi = torch.tensor([b for b, _ in heads])
    hi = torch.tensor([h for _, h in heads])
    sl = lambda t: t[bi, hi][None, :, :sample_tokens].contiguous()
    q, k, v, beta = (sl(x[n]) for n in ("q", "k", "v", "beta"))
    S0 = None if x.get("S0") is None else x["S0"][bi, hi][None].contiguous()
    oracle.recurrence(q[:, :1, :4], k[:, :1, :4], v[:, :1, :4], beta[:, :1, :4], threads=1)  # load
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.recurrence(q, k, v, beta, S0, threads=threads, want_o=True)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds or reps >= 1000:
            break
    return len(heads) * sample_tokens * reps / dt, dt, reps


def cpu_baseline_chunk(x, name, seconds=1.5):
    """The fp64 sequential oracle (C, OpenMP over (b, h)) on a bounded sample
    of workload ``x``: at all host threads on up to 64 (b, h) pairs, and at
    one thread on one pair.  tokens/s counts a token as one position of one
    batch row with all H heads, as the GPU figures do."""
    import oracle
    B, H, L, d = x["q"].shape
    nthreads = oracle.default_threads()
    pairs = [(b, h) for b in range(B) for h in range(H)][:64]
    T = max(64, min(L, int(2e9 / (len(pairs) * 6 * d * d * 4))))  # about 0.1-0.5 s per pass
    rate_n, dt_n, reps_n = oracle_rate(x, pairs, T, nthreads, seconds)
    T1 = max(64, min(L, int(4e8 / (6 * d * d))))
    rate_1, dt_1, reps_1 = oracle_rate(x, pairs[:1], T1, 1, seconds)
    used = min(nthreads, len(pairs))
    return {"value": rate_n / H, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"{name}: first {T} tokens of {len(pairs)} (b,h) pairs x{reps_n} ({dt_n:.1f} s), fp64 "
                      f"sequential recurrence, OpenMP over (b,h); head-tokens/s / H",
            "single_thread": {"value": rate_1 / H, "unit": "tokens/s", "cores": 1,
                              "sample": f"first {T1} tokens of 1 (b,h) pair x{reps_1} ({dt_1:.1f} s)"},
            "host_threads": nthreads, "cpu_model": cpu_model()}


def cpu_baseline_decode(seconds=1.5):
    """The fp64 oracle's one-token update on the decode batch (64 x 16 states,
    d = 128) from random states: all host threads on all 1024 states, one
    thread on 16 of them; tokens/s = batch rows per second."""
    import oracle
    Bd, Hd, d = workloads.DECODE_BATCH, workloads.DECODE_HEADS, 128
    xin = workloads.decode_inputs(1)
    S = workloads.random_state(Bd, Hd, d).double().numpy()
    nthreads = oracle.default_threads()
    out = {}
    for tag, nb, th in (("all", Bd, nthreads), ("one", 1, 1)):
        q, k, v, beta = (xin[n][0][:nb] for n in ("q", "k", "v", "beta"))
        Ss = S[:nb].copy()
        reps, t0 = 0, time.perf_counter()
        while True:
            _, Ss = oracle.decode_step(q, k, v, beta, Ss, threads=th)
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= seconds or reps >= 10000:
                break
        out[tag] = (nb * reps / dt, dt, reps)
    (rn, dtn, repn), (r1, dt1, rep1) = out["all"], out["one"]
    return {"value": rn, "unit": "tokens/s", "cores": min(nthreads, Bd * Hd), "kind": "oracle",
            "sample": f"decode: {Bd}x{Hd} states x{repn} steps ({dtn:.1f} s), fp64, OpenMP over (b,h)",
            "single_thread": {"value": r1, "unit": "tokens/s", "cores": 1,
                              "sample": f"1x{Hd} states x{rep1} steps ({dt1:.1f} s)"},
            "host_threads": nthreads, "cpu_model": cpu_model()}


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores, on the
    headline workload; each step is a bounded sample of it (the first 256
    tokens of every (b, h))."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    w = workloads.WORKLOADS[WORKLOAD]
    x = workloads.chunk_inputs(w)
    threads = oracle.default_threads()
    sample = 256
    q, k, v, beta = (x[n][:, :, :sample].contiguous() for n in ("q", "k", "v", "beta"))
    for _ in range(args.warmup):
        oracle.recurrence(q, k, v, beta, None, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.recurrence(q, k, v, beta, None, threads=threads)
    dt = time.perf_counter() - t0
    value = w.B * sample * args.steps / dt
    cores = min(threads, w.B * w.H)
    desc = (f"fp64 sequential oracle, first {sample} tokens of all {w.B}x{w.H} (b,h) of the {WORKLOAD} "
            f"workload per step, {cores} threads ({cpu_model()})")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": f"synthetic (seeded, workloads.{WORKLOAD} distribution)",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(w, n):
    s0 = "random S0" if w.s0 else "S0=0"
    return {"workload": f"{w.name}: B={w.B} H={w.H} L={w.L} d={w.d} C=64 {w.dtype} q/k/v, fp32 beta/state/o, {s0}",
            "B": w.B, "H": w.H, "L": w.L, "head_dim": w.d, "chunk": 64, "global_batch": w.B * n,
            "seq_len": w.L, "parallelism": f"dp{n} (independent (b,h) problems per rank, no collective)",
            "l2": "inputs and outputs (1.1 GB per call) exceed the 126 MB L2"}


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import delta_rule_linear_03_b200 as efla

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    w = workloads.WORKLOADS[WORKLOAD]
    B, H, L, d = w.B, w.H, w.L, w.d
    x = workloads.chunk_inputs(w, seed=rank_seed(w, rank))
    q, k, v, beta = (x[n].to(dev) for n in ("q", "k", "v", "beta"))
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=dev)
    S = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    ws = torch.empty(max(efla.workspace_size(q.dtype, B, H, L, d, d), 16), dtype=torch.uint8, device=dev)
    launches_per_step = chunk_launches(efla, q.dtype, B, H, L, d)
    stream = torch.cuda.current_stream(dev)
    call = lambda: efla.chunk_fwd(q, k, v, beta, None, o=o, S_L=S, workspace=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    g = graph_of(call)  # one call per replay keeps Python launch overhead off the clock
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    if efla.last_error() != 0:
        raise RuntimeError("efla_chunk_fwd reported a device-side error")

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index, period_s=0.001) as clk:
        barrier(world)
        torch.cuda.synchronize()
        clk.active.set()
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        clk.active.clear()
        barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world)
    ms_step = ms_max / args.steps
    value = job_tokens_per_s(world, B, L, args.steps, ms_max)
    del g

    nbytes = chunk_bytes(B, H, L, d, 2, 2, s0=False)  # o counted in the q dtype (bf16)
    nbytes_f32o = chunk_bytes(B, H, L, d, 2, 4, s0=False)
    flops = chunk_flops(B, H, L, d)
    achieved_tf = flops / (ms_step / 1e3) / 1e12
    roof = hbm_roofline(nbytes, ms_step, peaks, f"efla_chunk_fwd (all {launches_per_step} launches of one call)",
                        traffic=LONGCTX_TRAFFIC if WORKLOAD == "longctx" else None,
                        note="bytes count o in the q dtype (bf16), 1028 B per head-token; the call writes o "
                             "in fp32 (the default output dtype, 1284 B per head-token). traffic: DRAM bytes "
                             "of one call, 4 x an ncu capture at L = 16384 (same heads, same kernels)")
    roof["frac_with_fp32_o"] = nbytes_f32o / (ms_step / 1e3) / 1e9 / peaks["hbm"]

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": f"synthetic (seeded, workloads.{WORKLOAD} distribution)",
        "config": workload_config(w, world),
        "roofline": roof,
        "roofline_tensor": {"achieved": achieved_tf, "peak": peaks["bf16"], "unit": "TFLOP/s",
                            "frac": achieved_tf / peaks["bf16"], "algorithmic_flops": flops,
                            "peak_source": f"{peaks['source']} (cuBLAS bf16, burst)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_e2e:
        line["e2e"] = bench_e2e(efla, dev, x, args, world)
    del q, k, v, beta, o, S, ws
    torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_chunk(x, WORKLOAD)
    if rank == 0 and world == 1 and not args.no_configs:
        cfg = {"longctx_prefill": {"value": value / world, "unit": "tokens/s", "ms_per_call": ms_step,
                                   "config": line["config"]["workload"], "roofline": roof,
                                   "note": "the headline step", "cpu_baseline": line.get("cpu_baseline")}}
        for name in ("tiny_d32", "lm340m", "lm1p3b"):
            cfg[name] = bench_chunk_config(efla, dev, name, peaks, not args.no_cpu_baseline)
        cfg["stiffness"] = bench_stiffness(efla, dev, peaks, not args.no_cpu_baseline)
        cfg["longctx_decode"] = bench_decode(efla, dev, peaks, not args.no_cpu_baseline)
        line["configs"] = cfg
        line["deltanet_vs_efla"] = bench_modes(efla, dev)
        line["gate"] = bench_gate(efla, dev, peaks)
        if not args.no_backward:
            line["backward"] = bench_backward(efla, dev, peaks)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def chunk_case(efla, dev, name, rotate=1, mode="exact", **kw):
    """Device inputs, outputs and workspace of workload ``name`` (``rotate``
    independent sets when one set fits in L2) and a list of CUDA graphs of
    one efla_chunk_fwd call each."""
    sets, graphs = [], []
    for r in range(rotate):
        x = workloads.chunk_inputs(name, seed=None if r == 0 else 500 + r, **kw)
        B, H, L, d = x["q"].shape
        t = {n: (x[n].to(dev) if x[n] is not None else None) for n in ("q", "k", "v", "beta", "S0")}
        t["o"] = torch.empty(B, H, L, d, dtype=torch.float32, device=dev)
        t["S"] = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
        t["ws"] = torch.empty(max(efla.workspace_size(x["q"].dtype, B, H, L, d, d), 16), dtype=torch.uint8,
                              device=dev)
        sets.append(t)
    for t in sets:
        fn = lambda t=t: efla.chunk_fwd(t["q"], t["k"], t["v"], t["beta"], t["S0"], mode=mode, o=t["o"],
                                        S_L=t["S"], workspace=t["ws"])
        fn()
        torch.cuda.synchronize()
        graphs.append(graph_of(fn))
    return sets, graphs


def bench_chunk_config(efla, dev, name, peaks, with_cpu, reps=50):
    """efla_chunk_fwd on one workload at its full size: CUDA graph replays,
    rotating over independent input sets where one set fits in L2."""
    w = workloads.WORKLOADS[name]
    rotate = 3 if name == "lm340m" else 1
    sets, graphs = chunk_case(efla, dev, name, rotate=rotate)
    ms = time_replays(graphs, reps)
    if efla.last_error() != 0:
        raise RuntimeError("efla_chunk_fwd reported a device-side error")
    B, H, L, d = w.B, w.H, w.L, w.d
    es = 2 if w.dtype == "bf16" else 4
    out = {"value": B * L / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms, "calls": reps,
           "config": workload_config(w, 1)["workload"],
           "l2": (f"{rotate} rotating input/output sets (> L2)" if rotate > 1 else
                  ("inputs and outputs exceed L2" if name != "tiny_d32" else "L2-resident (0.3 MB): latency case")),
           "gpu_launches_per_call": chunk_launches(efla, w.torch_dtype, B, H, L, d)}
    if w.dtype == "bf16":
        out["roofline"] = hbm_roofline(chunk_bytes(B, H, L, d, es, es, s0=w.s0), ms, peaks,
                                       "efla_chunk_fwd (all launches of one call)",
                                       note="o counted in the q dtype; the call writes o in fp32")
        out["roofline"]["frac_with_fp32_o"] = chunk_bytes(B, H, L, d, es, 4, s0=w.s0) / (ms / 1e3) / 1e9 / peaks["hbm"]
    else:
        flops = chunk_flops(B, H, L, d)
        tf = flops / (ms / 1e3) / 1e12
        peak = ffma_peak_tflops(dev, peaks["sm_max_mhz"])
        out["roofline"] = {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                           "traffic": None, "kernel": "efla_chunk_fwd exact-fp32 path (all launches)",
                           "algorithmic_flops": flops,
                           "peak_source": "derived: SMs x 128 fp32 lanes x 2 flop x max SM clock"}
    del sets, graphs
    torch.cuda.empty_cache()
    if with_cpu:
        out["cpu_baseline"] = cpu_baseline_chunk(workloads.chunk_inputs(name), name)
    return out


def bench_modes(efla, dev, reps=20):
    """The pages' one throughput claim is that EFLA trains as fast as
    DeltaNet.  Both gates run through the same kernels here: the exact gate
    (EFLA) and alpha = beta (DeltaNet, explicit Euler), timed on lm340m and
    on the long-context prefill."""
    out = {}
    for name in ("lm340m", "longctx"):
        ms = {}
        for mode in ("exact", "euler"):
            sets, graphs = chunk_case(efla, dev, name, rotate=3 if name == "lm340m" else 1, mode=mode)
            ms[mode] = time_replays(graphs, reps)
            del sets, graphs
            torch.cuda.empty_cache()
        w = workloads.WORKLOADS[name]
        out[name] = {"efla_ms_per_call": ms["exact"], "deltanet_ms_per_call": ms["euler"],
                     "efla_tokens_per_s": w.B * w.L / (ms["exact"] / 1e3),
                     "deltanet_tokens_per_s": w.B * w.L / (ms["euler"] / 1e3),
                     "efla_over_deltanet_throughput": ms["euler"] / ms["exact"]}
    if efla.last_error() != 0:
        raise RuntimeError("efla_chunk_fwd reported a device-side error")
    return out


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

    block()
    torch.cuda.synchronize()
    ms = time_replays([graph_of(block)], reps) / 4
    rows = B * H * L
    nbytes = rows * (2 * d + 4 + 8)  # read k (bf16) and beta, write alpha and lambda
    return {"value": rows / (ms / 1e3), "unit": "keys/s", "ms_per_call": ms, "calls": 4 * reps,
            "config": f"lm1p3b keys: {B}x{H}x{L} rows of d={d} bf16, 4 rotating copies (> L2)",
            "roofline": hbm_roofline(nbytes, ms, peaks, "gate_kernel")}


def bench_backward(efla, dev, peaks, calls=5):
    """efla_prefill_bwd on lm340m (one fp32 dO, no S0/dS_L): exact fp32,
    one CTA per (b, h) walking the sequence three times."""
    x = workloads.chunk_inputs("lm340m")
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
    return {"value": B * L / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms, "calls": calls,
            "config": "lm340m backward: dq, dk, dv, dbeta, dS0 (fp32), bf16 q/k/v, fp32 dO",
            "kernel": "backward_kernel (fp32, serial over tokens per (b, h))"}


def bench_stiffness(efla, dev, peaks, with_cpu, calls=5):
    """The stiffness sweep on the exact-fp32 path: B=2, H=16, L=8192, d=128,
    fp32 q/k/v, ||k|| fixed per run at each of 1e-3, 0.1, 1, 10, 100.  One
    draw: the keys of each run are the unit keys times ||k||, the same fp32
    values the workload generator gives for that norm.  Inputs and outputs
    (0.5 GB) exceed L2; CUDA events over `calls` graph replays per norm.  The
    path is bound by fp32 arithmetic, so the roofline is the FFMA peak."""
    x = workloads.chunk_inputs("stiffness", knorm=1.0)
    q, k1, v, beta = (x[n].to(dev) for n in ("q", "k", "v", "beta"))
    B, H, L, d = k1.shape
    o = torch.empty(B, H, L, d, dtype=torch.float32, device=dev)
    S = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    ws = torch.empty(efla.workspace_size(q.dtype, B, H, L, d, d), dtype=torch.uint8, device=dev)
    per = {}
    for kn in workloads.STIFF_KNORMS:
        k = k1 * kn
        fn = lambda: efla.chunk_fwd(q, k, v, beta, None, o=o, S_L=S, workspace=ws)
        fn()
        per[kn] = time_replays([graph_of(fn)], calls)
        del k
    if efla.last_error() != 0:
        raise RuntimeError("efla_chunk_fwd reported a device-side error")
    ms = statistics.mean(per.values())
    flops = chunk_flops(B, H, L, d)
    tf = flops / (ms / 1e3) / 1e12
    peak = ffma_peak_tflops(dev, peaks["sm_max_mhz"])
    out = {"value": B * L / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms,
           "ms_per_knorm": {str(kn): t for kn, t in per.items()}, "calls": calls,
           "config": f"stiffness sweep: B={B} H={H} L={L} d={d} C=64 fp32 q/k/v/o/state, "
                     f"||k|| in {list(workloads.STIFF_KNORMS)}, beta ~ U(0,1), S0=0",
           "gpu_launches_per_call": 2,
           "roofline": {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                        "traffic": None, "kernel": "efla_chunk_fwd exact-fp32 path (all launches)",
                        "algorithmic_flops": flops,
                        "peak_source": "derived: SMs x 128 fp32 lanes x 2 flop x max SM clock"},
           "hbm_algorithmic_bytes": chunk_bytes(B, H, L, d, 4, 4, s0=False)}
    del q, k1, v, beta, o, S, ws
    torch.cuda.empty_cache()
    if with_cpu:
        out["cpu_baseline"] = cpu_baseline_chunk(x, "stiffness (||k|| = 1)")
    return out


def bench_decode(efla, dev, peaks, with_cpu, reps=3):
    """The long-context decode: 1024 chained efla_decode_step calls at batch
    64 x 16 heads x d = 128, fp32 states, bf16 q/k/v, fp32 o, captured as one
    CUDA graph of the 1024 steps.  The steps rotate over 4 state sets (256 MB,
    > L2), so every step reads and writes its state in HBM (4 interleaved
    chains of 256 steps); per-step inputs cycle over 64 drawn sets (0.6% of a
    step's bytes).  ``single_chain_l2_resident`` times one chain of 1024 steps
    on one 64 MB state set, which stays in the 126 MB L2 between steps."""
    Bd, Hd, d = workloads.DECODE_BATCH, workloads.DECODE_HEADS, 128
    steps, nsets, nin = workloads.DECODE_STEPS, 4, 64
    xin = workloads.decode_inputs(nin)
    ins = [{n: xin[n][i].to(dev) for n in ("q", "k", "v", "beta")} for i in range(nin)]
    states = [workloads.random_state(Bd, Hd, d, seed=s).to(dev) for s in range(nsets)]
    outs = [torch.empty(Bd, Hd, d, dtype=torch.float32, device=dev) for _ in range(nin)]

    def chain(rot):
        for i in range(steps):
            a = ins[i % nin]
            efla.decode_step(a["q"], a["k"], a["v"], a["beta"], states[i % rot], o=outs[i % nin])

    res = {}
    for rot in (nsets, 1):
        chain(rot)
        torch.cuda.synchronize()
        ms = time_replays([graph_of(lambda: chain(rot))], reps) / steps
        res[rot] = ms
    if efla.last_error() != 0:
        raise RuntimeError("efla_decode_step reported a device-side error")
    ms_step = res[nsets]
    nbytes = decode_bytes(Bd, Hd, d, 2, 4)
    out = {"value": Bd / (ms_step / 1e3), "unit": "tokens/s", "ms_per_step": ms_step,
           "steps_per_replay": steps, "replays": reps,
           "config": f"batch {Bd} x {Hd} heads x d={d}, fp32 states, bf16 q/k/v, fp32 o; one CUDA graph of "
                     f"{steps} steps over {nsets} rotating state sets (> L2)",
           "gpu_launches_per_replay": steps,
           "roofline": hbm_roofline(nbytes, ms_step, peaks, "decode_kernel"),
           "single_chain_l2_resident": {"value": Bd / (res[1] / 1e3), "unit": "tokens/s", "ms_per_step": res[1],
                                        "note": "one 64 MB state set: L2-resident between steps"}}
    del ins, states, outs
    torch.cuda.empty_cache()
    if with_cpu:
        out["cpu_baseline"] = cpu_baseline_decode()
    return out


def bench_e2e(efla, dev, x, args, world):
    """The same metric through the public API from pinned host buffers:
    every step copies q, k, v, beta host->device, runs efla_chunk_fwd and
    copies o and S_L device->host.  Steps are pipelined the way a serving
    loop would run them: three streams (copy in, compute, copy out) and two
    device buffer sets, so that step i+1's inputs cross PCIe while step i
    computes and step i-1's outputs come back (PCIe is full duplex).  Each
    step still moves all of its own inputs and outputs inside the timed
    region; a buffer set is refilled only after the step that used it has
    been copied out."""
    hq, hk, hv, hb = (x[n].pin_memory() for n in ("q", "k", "v", "beta"))
    B, H, L, d = hq.shape
    ho = [torch.empty(B, H, L, d, dtype=torch.float32).pin_memory() for _ in range(2)]
    hS = [torch.empty(B, H, d, d, dtype=torch.float32).pin_memory() for _ in range(2)]
    din = [tuple(torch.empty_like(t, device=dev) for t in (hq, hk, hv, hb)) for _ in range(2)]
    do = [torch.empty(B, H, L, d, dtype=torch.float32, device=dev) for _ in range(2)]
    dS = [torch.empty(B, H, d, d, dtype=torch.float32, device=dev) for _ in range(2)]
    ws = torch.empty(max(efla.workspace_size(hq.dtype, B, H, L, d, d), 16), dtype=torch.uint8, device=dev)
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[b])       # step i-2 has finished reading this input set
            for dst, src in zip(din[b], (hq, hk, hv, hb)):
                dst.copy_(src, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            s_comp.wait_event(ev_out[b])      # step i-2's outputs have left this output set
            efla.chunk_fwd(*din[b], None, o=do[b], S_L=dS[b], workspace=ws)
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            ho[b].copy_(do[b], non_blocking=True)
            hS[b].copy_(dS[b], non_blocking=True)
            ev_out[b].record(s_out)

    def run(n):
        cur = torch.cuda.current_stream(dev)
        for s in (s_in, s_comp, s_out):
            s.wait_stream(cur)
        for i in range(n):
            step(i)
        for s in (s_in, s_comp, s_out):
            cur.wait_stream(s)

    run(3)
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record()
    run(n)
    e1.record()
    torch.cuda.synchronize()
    if efla.last_error() != 0:
        raise RuntimeError("efla_chunk_fwd reported a device-side error")
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    barrier(world)
    e0.record()
    run(1)                                     # one step alone: its latency, copies included
    e1.record()
    torch.cuda.synchronize()
    one_ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hb))
    d2h = ho[0].numel() * ho[0].element_size() + hS[0].numel() * hS[0].element_size()
    return {"value": world * B * L * n / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "ms_per_step": ms / n, "single_step_ms": one_ms,
            "pipeline": "3 streams (copy in / compute / copy out), 2 buffer sets; steps overlap"}


def run_profile_case(case: str, calls: int, seq_len=None):
    """A few plain calls of one kernel's workload and nothing else, for an
    ncu capture of that kernel (no timing, no output line).  ``seq_len``
    shortens a prefill workload (same heads, same kernels) for captures
    that would be too large at full length."""
    import delta_rule_linear_03_b200 as efla
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if case == "gate":
        x = workloads.chunk_inputs("lm1p3b")
        k, beta = x["k"].to(dev), x["beta"].to(dev)
        for _ in range(calls):
            efla.gate(k, beta)
    elif case == "decode":
        Bd, Hd, d = workloads.DECODE_BATCH, workloads.DECODE_HEADS, 128
        xin = workloads.decode_inputs(calls)
        states = [workloads.random_state(Bd, Hd, d, seed=s).to(dev) for s in range(4)]
        for i in range(calls):
            efla.decode_step(*(xin[n][i].to(dev) for n in ("q", "k", "v", "beta")), states[i % 4])
    else:
        x = workloads.chunk_inputs(case, L=seq_len)
        t = {n: (x[n].to(dev) if x[n] is not None else None) for n in ("q", "k", "v", "beta", "S0")}
        for _ in range(calls):
            efla.chunk_fwd(t["q"], t["k"], t["v"], t["beta"], t["S0"])
    torch.cuda.synchronize()
    if efla.last_error() != 0:
        raise RuntimeError("device-side error")
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="headline only")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--profile-case", choices=["gate", "decode", "tiny_d32", "lm340m", "lm1p3b", "stiffness",
                                               "longctx"],
                    help="run a few plain calls of one workload for an ncu capture, then exit")
    ap.add_argument("--calls", type=int, default=4, help="calls for --profile-case")
    ap.add_argument("--profile-len", type=int, default=None, help="sequence length for --profile-case")
    args = ap.parse_args(argv)
    if args.profile_case:
        return run_profile_case(args.profile_case, args.calls, args.profile_len)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
