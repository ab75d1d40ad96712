"""Seeded synthetic inputs for the EFLA token mixer.

This module is shared by the tests, the smoke check and the benchmark, for
both the CUDA path and the oracle.  It holds none of the method's
arithmetic: it only draws random numbers, normalises vectors and rounds them
to the storage dtype.  Both sides read exactly the arrays it returns (bf16
values widen exactly to fp32/fp64).

Workloads (shapes and value distributions):

* ``tiny_d32``   B=1 H=2 L=256 d=32, fp32.  q,k,v ~ N(0,1); beta=sigmoid(N(0,1)); S0=0.
* ``lm340m``     B=8 H=8 L=2048 d=128, bf16 q/k/v.  q,k,v ~ N(0,1/128); q
  L2-normalised per (b,h,t); k L2-normalised then scaled by s ~ LogNormal(0,0.5)
  drawn per (b,h,t); beta=sigmoid(N(0,1)) fp32; S0=0.
* ``lm1p3b``     B=4 H=16 L=4096 d=128, bf16, as lm340m; S0 ~ N(0, 0.01) fp32.
* ``stiffness``  B=2 H=16 L=8192 d=128, fp32.  ||k|| fixed per run in
  {1e-3, 0.1, 1, 10, 100} with a uniformly random direction; beta ~ U(0,1);
  q, v as lm340m (fp32).  S0=0.
* ``longctx``    B=1 H=16 L=65536 d=128, bf16 prefill as lm340m; then decode
  steps at batch 64 x 16 heads with fresh q/k/v/beta per step drawn as lm340m
  (step s from its own generator, see ``decode_inputs``).

Seeds: ``numpy.random.default_rng(42 + index)`` with index the workload's
position in ``WORKLOADS``; draw order q, k, v, key-norm scales, beta, S0.
Every generator accepts reduced B/H/L for tests that need small cases of the
same distribution.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch

CHUNK = 64


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    H: int
    L: int
    d: int
    dtype: str          # "f32" or "bf16": storage dtype of q, k, v, o
    kind: str           # "gauss" | "lm" | "stiff"
    s0: bool = False    # random initial state
    knorm: float | None = None

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny_d32": Workload("tiny_d32", 0, 1, 2, 256, 32, "f32", "gauss"),
    "lm340m": Workload("lm340m", 1, 8, 8, 2048, 128, "bf16", "lm"),
    "lm1p3b": Workload("lm1p3b", 2, 4, 16, 4096, 128, "bf16", "lm", s0=True),
    "stiffness": Workload("stiffness", 3, 2, 16, 8192, 128, "f32", "stiff", knorm=1.0),
    "longctx": Workload("longctx", 4, 1, 16, 65536, 128, "bf16", "lm"),
}
STIFF_KNORMS = (1e-3, 0.1, 1.0, 10.0, 100.0)
DECODE_BATCH = 64
DECODE_HEADS = 16
DECODE_STEPS = 1024


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _unit(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    n[n == 0] = 1.0
    return (x / n).astype(np.float32)


def _to(x: np.ndarray, dtype) -> torch.Tensor:
    """Round (nearest-even) to the storage dtype on the host."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype)


def _draw_qkv(rng, kind, B, H, L, d, knorm):
    shp = (B, H, L, d)
    if kind == "gauss":
        q = rng.standard_normal(shp, dtype=np.float32)
        k = rng.standard_normal(shp, dtype=np.float32)
        v = rng.standard_normal(shp, dtype=np.float32)
        beta = _sigmoid(rng.standard_normal((B, H, L), dtype=np.float32))
        return q, k, v, beta
    sd = np.float32(1.0 / np.sqrt(128.0))
    q = rng.standard_normal(shp, dtype=np.float32) * sd
    k = rng.standard_normal(shp, dtype=np.float32) * sd
    v = rng.standard_normal(shp, dtype=np.float32) * sd
    q = _unit(q)
    if kind == "lm":
        s = np.exp(0.5 * rng.standard_normal((B, H, L, 1), dtype=np.float32)).astype(np.float32)
        k = _unit(k) * s
        beta = _sigmoid(rng.standard_normal((B, H, L), dtype=np.float32))
    elif kind == "stiff":
        k = _unit(k) * np.float32(knorm)
        beta = rng.uniform(0.0, 1.0, (B, H, L)).astype(np.float32)
    else:
        raise ValueError(kind)
    return q, k, v, beta


def chunk_inputs(w: Workload | str, *, B=None, H=None, L=None, knorm=None, seed=None,
                 s0=None, dtype=None):
    """Inputs of ``efla_chunk_fwd`` for workload ``w`` as CPU torch tensors:
    dict(q, k, v [B,H,L,d] storage dtype; beta [B,H,L] fp32; S0 [B,H,d,d] fp32 or None).
    ``dtype`` ("f32" or "bf16") overrides the workload's storage dtype; the
    values are drawn the same way and then rounded to it."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if dtype is not None:
        w = w.with_(dtype=dtype)
    B = w.B if B is None else B
    H = w.H if H is None else H
    L = w.L if L is None else L
    knorm = w.knorm if knorm is None else knorm
    use_s0 = w.s0 if s0 is None else s0
    rng = np.random.default_rng(42 + w.index if seed is None else seed)
    q, k, v, beta = _draw_qkv(rng, w.kind, B, H, L, w.d, knorm)
    S0 = None
    if use_s0:
        S0 = torch.from_numpy(rng.standard_normal((B, H, w.d, w.d), dtype=np.float32) * np.float32(0.1))
    dt = w.torch_dtype
    return dict(q=_to(q, dt), k=_to(k, dt), v=_to(v, dt), beta=torch.from_numpy(beta),
                S0=S0)


def decode_inputs(steps: int, *, B=DECODE_BATCH, H=DECODE_HEADS, d=128, dtype="bf16",
                  first: int = 0, seed=None):
    """Per-step decode inputs drawn as lm340m: q,k,v [steps,B,H,d], beta
    [steps,B,H], for the steps first .. first+steps-1 of the decode stream.
    Step s is drawn from its own generator, ``default_rng([base, s])`` with
    base = 42 + longctx index + 1000, so any window of a long chain (the
    1024-step long-context decode) is generated without the steps before it."""
    base = 42 + WORKLOADS["longctx"].index + 1000 if seed is None else seed
    qs, ks, vs, bs = [], [], [], []
    for s in range(first, first + steps):
        rng = np.random.default_rng([base, s])
        q, k, v, beta = _draw_qkv(rng, "lm", 1, B, H, d, None)  # [1,B,H,d]: one "token" per state
        qs.append(q.reshape(B, H, d))
        ks.append(k.reshape(B, H, d))
        vs.append(v.reshape(B, H, d))
        bs.append(beta.reshape(B, H))
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    return dict(q=_to(np.stack(qs), dt), k=_to(np.stack(ks), dt), v=_to(np.stack(vs), dt),
                beta=torch.from_numpy(np.stack(bs)))


def random_state(B, H, d, std=0.1, seed=7):
    """A random fp32 state [B,H,d,d] ~ N(0, std^2)."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal((B, H, d, d), dtype=np.float32) * np.float32(std))
