"""fp64 CPU oracle for the EFLA token mixer.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``delta_rule_linear_03_b200``) never imports it,
and the two share no code: this package wraps the plain C file
``efla_oracle.c`` (compiled with gcc, no GPU) through ctypes.

What the functions compute, with the passages they follow ("Exact Flow
Linear Attention: Exact Solution from Continuous-Time Dynamics",
papernotes.org summary of arXiv 2512.12602):

* ``alpha`` / ``gate`` - the exact-flow gate of section 关键设计 2,
  alpha = (1 - e^{-beta*lambda}) / lambda with lambda = ||k||^2, evaluated as
  -expm1(-beta*lambda_c)/lambda_c with lambda_c = max(lambda, 1e-12)
  (section 损失函数 / 训练策略).  ``euler=True`` gives the DeltaNet step
  alpha = beta (section 关键设计 1).
* ``recurrence`` - the sequential update S_t = (I - alpha k k^T) S_{t-1} +
  alpha k v^T and readout o_t = S_t^T q_t (关键设计 2, flowchart of 整体框架).
  This is the oracle the CUDA path is compared against.
* ``chunked`` - the same recurrence through the chunked UT form (整体框架:
  chunks of size C), used only to check that algebra against ``recurrence``.
* ``expm_taylor``, ``duhamel``, ``rk4_step`` - brute-force matrix exponential,
  Gauss-Legendre quadrature of the Duhamel integral, and the RK4
  specialisation of the jsqmd.com blog section 5.3; these pin the oracle to
  the ODE without using the closed form.

All arrays are float64, C-contiguous, row-major.  Every function is pinned by
tests in ``tests/test_oracle_pins.py``; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "efla_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_SO = os.path.join(_OUT_DIR, "libefla_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``efla_oracle.c`` into ``_build/libefla_oracle.so`` with gcc."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_SO)
            and os.path.getmtime(_SO) >= os.path.getmtime(_SRC)):
        return _SO
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        # EFLA_ORACLE_SO lets the mutation test load a deliberately broken
        # copy of this oracle to check that the pins notice.
        lib = ctypes.CDLL(os.environ.get("EFLA_ORACLE_SO") or build())
        d, i, l, p = ctypes.c_double, ctypes.c_int, ctypes.c_long, ctypes.c_void_p
        lib.efla_oracle_alpha.restype = d
        lib.efla_oracle_alpha.argtypes = [d, d, i]
        lib.efla_oracle_gate.restype = None
        lib.efla_oracle_gate.argtypes = [p, p, l, i, i, p, p]
        lib.efla_oracle_recurrence.restype = None
        lib.efla_oracle_recurrence.argtypes = [p, p, p, p, p, i, i, i, i, i, i, p, p, i]
        lib.efla_oracle_chunked.restype = None
        lib.efla_oracle_chunked.argtypes = [p, p, p, p, p, i, i, i, i, i, i, i, p, p, i]
        lib.efla_oracle_backward.restype = None
        lib.efla_oracle_backward.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, i, p, p, p, p, p, i]
        lib.efla_oracle_expm_taylor.restype = None
        lib.efla_oracle_expm_taylor.argtypes = [i, p, d, p]
        lib.efla_oracle_duhamel.restype = None
        lib.efla_oracle_duhamel.argtypes = [i, i, p, p, d, i, p]
        lib.efla_oracle_rk4_step.restype = None
        lib.efla_oracle_rk4_step.argtypes = [i, i, p, p, d, p, p]
        _lib = lib
        return lib


def _f64(x) -> np.ndarray:
    """Widen any array-like (numpy, or a CPU torch tensor of any float dtype)
    to a C-contiguous float64 numpy array.  bf16/fp32 widen exactly."""
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def alpha(beta: float, lam: float, euler: bool = False) -> float:
    return _load().efla_oracle_alpha(float(beta), float(lam), int(euler))


def gate(k, beta, euler: bool = False):
    """k [..., dk], beta [...] -> (alpha, lambda), both shaped like beta."""
    k = _f64(k)
    beta = _f64(beta)
    dk = k.shape[-1]
    rows = int(np.prod(k.shape[:-1]))
    assert beta.size == rows
    a = np.empty(rows)
    lam = np.empty(rows)
    _load().efla_oracle_gate(_ptr(k), _ptr(beta), rows, dk, int(euler), _ptr(a), _ptr(lam))
    return a.reshape(beta.shape), lam.reshape(beta.shape)


def _prep(q, k, v, beta, S0):
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    B, H, L, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, H, L) and beta.shape == (B, H, L)
    if S0 is not None:
        S0 = _f64(S0)
        assert S0.shape == (B, H, dk, dv)
    return q, k, v, beta, S0, B, H, L, dk, dv


def recurrence(q, k, v, beta, S0=None, euler: bool = False, threads: int | None = None,
               want_o: bool = True):
    """Sequential fp64 recurrence. q,k [B,H,L,dk], v [B,H,L,dv], beta [B,H,L],
    S0 [B,H,dk,dv] or None.  Returns (o [B,H,L,dv] or None, S_L [B,H,dk,dv])."""
    q, k, v, beta, S0, B, H, L, dk, dv = _prep(q, k, v, beta, S0)
    o = np.empty((B, H, L, dv)) if want_o else None
    SL = np.empty((B, H, dk, dv))
    _load().efla_oracle_recurrence(
        _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0) if S0 is not None else None,
        B, H, L, dk, dv, int(euler), _ptr(o) if o is not None else None, _ptr(SL),
        threads or default_threads())
    return o, SL


def backward(q, k, v, beta, S0, dO, dSL=None, euler: bool = False, threads: int | None = None):
    """Reverse-mode derivative of ``recurrence`` for the loss
    L = sum(dO * o) + sum(dSL * S_L): returns (dq, dk, dv, dbeta, dS0) in fp64."""
    q, k, v, beta, S0, B, H, L, dk, dv = _prep(q, k, v, beta, S0)
    dO = _f64(dO)
    assert dO.shape == (B, H, L, dv)
    if dSL is not None:
        dSL = _f64(dSL)
        assert dSL.shape == (B, H, dk, dv)
    dq, dkk = np.empty((B, H, L, dk)), np.empty((B, H, L, dk))
    dvv, dbeta, dS0 = np.empty((B, H, L, dv)), np.empty((B, H, L)), np.empty((B, H, dk, dv))
    _load().efla_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0) if S0 is not None else None, _ptr(dO),
        _ptr(dSL) if dSL is not None else None, B, H, L, dk, dv, int(euler),
        _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dbeta), _ptr(dS0), threads or default_threads())
    return dq, dkk, dvv, dbeta, dS0


def chunked(q, k, v, beta, S0=None, C: int = 64, euler: bool = False,
            threads: int | None = None):
    """Chunked UT-form fp64 evaluation of the same recurrence."""
    q, k, v, beta, S0, B, H, L, dk, dv = _prep(q, k, v, beta, S0)
    o = np.empty((B, H, L, dv))
    SL = np.empty((B, H, dk, dv))
    _load().efla_oracle_chunked(
        _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(S0) if S0 is not None else None,
        B, H, L, dk, dv, int(C), int(euler), _ptr(o), _ptr(SL), threads or default_threads())
    return o, SL


def decode_step(q, k, v, beta, S, euler: bool = False, threads: int | None = None):
    """One-token update of states S [B,H,dk,dv] with q,k [B,H,dk], v [B,H,dv],
    beta [B,H]: the recurrence at L=1.  Returns (o [B,H,dv], S_new)."""
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    o, SL = recurrence(q[:, :, None], k[:, :, None], v[:, :, None], beta[:, :, None],
                       S, euler=euler, threads=threads)
    return o[:, :, 0], SL


def expm_taylor(M, t: float = 1.0):
    """e^{tM} by brute-force Taylor series with scaling and squaring."""
    M = _f64(M)
    d = M.shape[0]
    out = np.empty((d, d))
    _load().efla_oracle_expm_taylor(d, _ptr(M), float(t), _ptr(out))
    return out


def duhamel(k, v, beta: float, panels: int = 64):
    """int_0^beta e^{-(beta-tau) k k^T} k v^T dtau by Gauss-Legendre quadrature."""
    k, v = _f64(k), _f64(v)
    out = np.empty((k.size, v.size))
    _load().efla_oracle_duhamel(k.size, v.size, _ptr(k), _ptr(v), float(beta), int(panels),
                                _ptr(out))
    return out


def rk4_step(k, v, beta: float, S):
    """The RK4 specialisation of one ZOH step (jsqmd.com blog, section 5.3)."""
    k, v, S = _f64(k), _f64(v), _f64(S)
    out = np.empty_like(S)
    _load().efla_oracle_rk4_step(k.size, v.size, _ptr(k), _ptr(v), float(beta), _ptr(S),
                                 _ptr(out))
    return out
