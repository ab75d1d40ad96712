"""EFLA (Exact Flow Linear Attention) token mixer on B200 (sm_100a).

Thin Python binding over the C ABI of ``include/efla.h`` (``libefla.so``,
built in-tree by ``delta_rule_linear_03_b200/build.py``).  This module only
marshals arguments: it checks devices, dtypes and contiguity, allocates
outputs and scratch with PyTorch, and passes raw device pointers and the
current CUDA stream.  Every step of the computation runs in the library's
CUDA kernels; there is no CPU fallback, and importing this module fails
loudly when the library is missing.

    o, S_L = chunk_fwd(q, k, v, beta, S0=None)      # prefill, [B,H,L,d]
    o      = decode_step(q, k, v, beta, S)          # S updated in place
    alpha, lam = gate(k, beta)

The method ("Exact Flow Linear Attention: Exact Solution from Continuous-Time
Dynamics", papernotes.org summary of arXiv 2512.12602, 关键设计 2):
S_t = (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T, o_t = S_t^T q_t,
alpha_t = (1 - e^{-beta_t ||k_t||^2}) / ||k_t||^2.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libefla.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python delta_rule_linear_03_b200/build.py` "
        "(nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

EFLA_F32, EFLA_BF16 = 0, 1
MODES = {"exact": 0, "euler": 1}
STATUS = {0: "EFLA_OK", 1: "EFLA_ERR_NULL", 2: "EFLA_ERR_SHAPE", 3: "EFLA_ERR_DTYPE", 4: "EFLA_ERR_ALIGN",
          5: "EFLA_ERR_UNSUPPORTED", 6: "EFLA_ERR_CUDA", 7: "EFLA_ERR_TIMEOUT", 8: "EFLA_ERR_WORKSPACE",
          9: "EFLA_ERR_ALIAS"}
EXPORTS = ("efla_status_string", "efla_version", "efla_last_error", "efla_gate",
           "efla_chunk_fwd_workspace_size", "efla_chunk_fwd", "efla_decode_step",
           "efla_chunk_fwd_workspace_size_simt", "efla_chunk_fwd_noalloc", "efla_diag_wait_timeout",
           "efla_state_affine", "efla_prefill_bwd_workspace_size", "efla_prefill_bwd")
NOALLOC_SCRATCH_BYTES = 32 << 20

_p, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_lib.efla_status_string.restype = ctypes.c_char_p
_lib.efla_status_string.argtypes = [_i]
_lib.efla_version.restype = _i
_lib.efla_version.argtypes = []
_lib.efla_last_error.restype = _i
_lib.efla_last_error.argtypes = []
_lib.efla_gate.restype = _i
_lib.efla_gate.argtypes = [_p, _i, _i, _p, _p, _p, _i, _i, _i, _i, _p]
_lib.efla_chunk_fwd_workspace_size.restype = _sz
_lib.efla_chunk_fwd_workspace_size.argtypes = [_i, _i, _i, _i, _i, _i]
_lib.efla_chunk_fwd.restype = _i
_lib.efla_chunk_fwd.argtypes = [_p, _p, _p, _i, _i, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _p, _sz, _p]
_lib.efla_chunk_fwd_workspace_size_simt.restype = _sz
_lib.efla_chunk_fwd_workspace_size_simt.argtypes = [_i, _i, _i, _i, _i]
_lib.efla_chunk_fwd_noalloc.restype = _i
_lib.efla_chunk_fwd_noalloc.argtypes = [_p, _p, _p, _i, _i, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _p]
_lib.efla_diag_wait_timeout.restype = _i
_lib.efla_diag_wait_timeout.argtypes = [ctypes.c_longlong, _p]
_lib.efla_decode_step.restype = _i
_lib.efla_decode_step.argtypes = [_p, _p, _p, _i, _i, _p, _p, _p, _i, _i, _i, _i, _i, _p]
_lib.efla_state_affine.restype = _i
_lib.efla_state_affine.argtypes = [_p, _p, _p, _p, _i, _i, _i, _p]
_lib.efla_prefill_bwd_workspace_size.restype = _sz
_lib.efla_prefill_bwd_workspace_size.argtypes = [_i, _i, _i, _i, _i]
_lib.efla_prefill_bwd.restype = _i
_lib.efla_prefill_bwd.argtypes = [_p, _p, _p, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                                  _i, _i, _i, _i, _i, _p, _sz, _p]


class EflaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.efla_status_string(status).decode()
        super().__init__(f"{where}: {msg}")


def _check(status: int, where: str):
    if status != 0:
        raise EflaError(status, where)


def _dt(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return EFLA_F32
    if x.dtype == torch.bfloat16:
        return EFLA_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {x.dtype}")


def _dev(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must be on one device")
    return dev


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def version() -> int:
    return _lib.efla_version()


def last_error() -> int:
    """Synchronise and return the sticky device status (0 = EFLA_OK)."""
    return _lib.efla_last_error()


def gate(k: torch.Tensor, beta: torch.Tensor, mode: str = "exact", alpha=None, lam=None):
    """k [B,H,L,d_k] (fp32/bf16), beta [B,H,L] fp32 -> (alpha, lambda) fp32 [B,H,L]."""
    dev = _dev(k, beta)
    B, H, L, dk = k.shape
    if beta.dtype != torch.float32 or tuple(beta.shape) != (B, H, L):
        raise ValueError("beta must be float32 [B,H,L]")
    alpha = torch.empty((B, H, L), dtype=torch.float32, device=dev) if alpha is None else alpha
    lam = torch.empty((B, H, L), dtype=torch.float32, device=dev) if lam is None else lam
    for t in (alpha, lam):
        if t.dtype != torch.float32 or tuple(t.shape) != (B, H, L):
            raise ValueError("alpha and lambda must be float32 [B,H,L]")
    _dev(k, alpha, lam)
    with torch.cuda.device(dev):
        _check(_lib.efla_gate(_ptr(k), _dt(k), MODES[mode], _ptr(beta), _ptr(alpha), _ptr(lam),
                              B, H, L, dk, _stream(dev)), "efla_gate")
    return alpha, lam


def workspace_size(dtype: torch.dtype, B: int, H: int, L: int, d_k: int, d_v: int) -> int:
    dt = EFLA_F32 if dtype == torch.float32 else EFLA_BF16
    return int(_lib.efla_chunk_fwd_workspace_size(dt, B, H, L, d_k, d_v))


def _prefill_args(q, k, v, beta, S0, o, S_L, want_state, out_dtype):
    """Shape and dtype checks shared by both prefill entry points; returns
    (device, B, H, L, d_k, d_v, o, S_L) with the outputs allocated when not
    given.  The C ABI sizes every buffer from B, H, L and d, so a caller
    buffer of the wrong shape or dtype is refused here, before any launch."""
    dev = _dev(q, k, v, beta, S0)
    if k.dim() != 4:
        raise ValueError("q, k, v must be [B,H,L,d]")
    B, H, L, dk = k.shape
    dv = v.shape[-1]
    if q.shape != k.shape or v.dim() != 4 or v.shape[:3] != (B, H, L) or q.dtype != k.dtype or v.dtype != k.dtype:
        raise ValueError("q, k, v must share dtype and [B,H,L,*] shape")
    _dt(q)
    if beta.dtype != torch.float32 or tuple(beta.shape) != (B, H, L):
        raise ValueError("beta must be float32 [B,H,L]")
    if S0 is not None and (S0.dtype != torch.float32 or tuple(S0.shape) != (B, H, dk, dv)):
        raise ValueError("S0 must be float32 [B,H,d_k,d_v]")
    if o is None:
        o = torch.empty((B, H, L, dv), dtype=out_dtype, device=dev)
    if tuple(o.shape) != (B, H, L, dv) or o.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("o must be float32 or bfloat16 [B,H,L,d_v]")
    if want_state and S_L is None:
        S_L = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if S_L is not None and (S_L.dtype != torch.float32 or tuple(S_L.shape) != (B, H, dk, dv)):
        raise ValueError("S_L must be float32 [B,H,d_k,d_v]")
    _dev(q, o, S_L)
    return dev, B, H, L, dk, dv, o, S_L


def chunk_fwd(q, k, v, beta, S0=None, mode: str = "exact", o=None, S_L=None, want_state: bool = True,
              workspace=None, out_dtype=torch.float32):
    """Prefill: q,k [B,H,L,d_k], v [B,H,L,d_v] (one dtype, fp32 or bf16), beta [B,H,L]
    fp32, S0 [B,H,d_k,d_v] fp32 or None.  Returns (o [B,H,L,d_v] in ``out_dtype``
    (or ``o.dtype`` when ``o`` is given), S_L [B,H,d_k,d_v] fp32 or None).
    ``S_L=S0`` updates the state in place."""
    dev, B, H, L, dk, dv, o, S_L = _prefill_args(q, k, v, beta, S0, o, S_L, want_state, out_dtype)
    need = workspace_size(q.dtype, B, H, L, dk, dv)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(_lib.efla_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _dt(q), MODES[mode], _ptr(beta), _ptr(S0),
                                   _ptr(o), _dt(o), _ptr(S_L), B, H, L, dk, dv,
                                   _ptr(workspace) if need else None, wbytes if need else 0,
                                   _stream(dev)), "efla_chunk_fwd")
    return o, S_L


def chunk_fwd_noalloc(q, k, v, beta, S0=None, mode: str = "exact", o=None, S_L=None,
                      want_state: bool = True, out_dtype=torch.float32):
    """``chunk_fwd`` through the entry point that allocates no device memory
    (its scratch is a fixed 32 MiB array inside the library, shared by all
    calls on a device; calls that overlap on the GPU race on it).  For hosts
    that cannot let a library allocate.  Outputs are allocated here only when
    not passed in."""
    dev, B, H, L, dk, dv, o, S_L = _prefill_args(q, k, v, beta, S0, o, S_L, want_state, out_dtype)
    with torch.cuda.device(dev):
        _check(_lib.efla_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _dt(q), MODES[mode], _ptr(beta),
                                           _ptr(S0), _ptr(o), _dt(o), _ptr(S_L), B, H, L, dk, dv,
                                           _stream(dev)), "efla_chunk_fwd_noalloc")
    return o, S_L


def decode_step(q, k, v, beta, S, mode: str = "exact", o=None, out_dtype=torch.float32):
    """One token for B*H states: q,k [B,H,d_k], v [B,H,d_v], beta [B,H] fp32,
    S [B,H,d_k,d_v] fp32 updated in place.  Returns o [B,H,d_v] in ``out_dtype``
    (or ``o.dtype`` when ``o`` is given)."""
    dev = _dev(q, k, v, beta, S)
    B, H, dk = k.shape
    dv = v.shape[-1]
    if q.shape != k.shape or v.shape[:2] != (B, H) or q.dtype != k.dtype or v.dtype != k.dtype:
        raise ValueError("q, k, v must share dtype and [B,H,*] shape")
    if beta.dtype != torch.float32 or tuple(beta.shape) != (B, H):
        raise ValueError("beta must be float32 [B,H]")
    if S.dtype != torch.float32 or tuple(S.shape) != (B, H, dk, dv):
        raise ValueError("S must be float32 [B,H,d_k,d_v]")
    o = torch.empty((B, H, dv), dtype=out_dtype, device=dev) if o is None else o
    if tuple(o.shape) != (B, H, dv):
        raise ValueError("o must be [B,H,d_v]")
    _dev(o)
    with torch.cuda.device(dev):
        _check(_lib.efla_decode_step(_ptr(q), _ptr(k), _ptr(v), _dt(q), MODES[mode], _ptr(beta), _ptr(S),
                                     _ptr(o), _dt(o), B, H, dk, dv, _stream(dev)), "efla_decode_step")
    return o


def state_affine(SI, SZ, X, out=None):
    """(SI - SZ) @ X + SZ for every (b, h): [B,H,d,d] fp32, d in {32, 64, 128}.
    With SI / SZ the final states of a segment from the identity / from zero
    and X the segment's true initial state, the result is its true final
    state (the state map of a segment is affine)."""
    dev = _dev(SI, SZ, X, out)
    for t in (SI, SZ, X):
        if t.dtype != torch.float32 or t.dim() != 4 or t.shape != SI.shape or not t.is_contiguous():
            raise ValueError("SI, SZ, X must be contiguous float32 [B,H,d,d] of one shape")
    B, H, d, d2 = SI.shape
    if d != d2:
        raise ValueError("square states only")
    if out is None:
        out = torch.empty_like(SI)
    elif out.dtype != torch.float32 or out.shape != SI.shape:
        raise ValueError("out must be float32 [B,H,d,d]")
    with torch.cuda.device(dev):
        _check(_lib.efla_state_affine(_ptr(SI), _ptr(SZ), _ptr(X), _ptr(out), B, H, d, _stream(dev)),
               "efla_state_affine")
    return out


def prefill_bwd(q, k, v, beta, S0, dO, dSL=None, mode: str = "exact", workspace=None):
    """Gradients of L = sum(dO * o) + sum(dSL * S_L) for ``chunk_fwd(q, k, v,
    beta, S0)``: returns (dq, dk, dv [B,H,L,d], dbeta [B,H,L], dS0 [B,H,d,d]),
    all float32.  q, k, v share one dtype (fp32 or bf16); beta, S0 (or
    None), dO and dSL (or None) are float32."""
    dev = _dev(q, k, v, beta, S0, dO, dSL)
    B, H, L, dk_ = k.shape
    dv_ = v.shape[-1]
    if q.shape != k.shape or v.shape[:3] != (B, H, L) or q.dtype != k.dtype or v.dtype != k.dtype:
        raise ValueError("q, k, v must share dtype and [B,H,L,*] shape")
    for name, t, shape in (("beta", beta, (B, H, L)), ("dO", dO, (B, H, L, dv_)),
                           ("S0", S0, (B, H, dk_, dv_)), ("dSL", dSL, (B, H, dk_, dv_))):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous()):
            raise ValueError(f"{name} must be contiguous float32 {shape}")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    f = dict(dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty(B, H, L, dk_, **f), torch.empty(B, H, L, dk_, **f), torch.empty(B, H, L, dv_, **f)
    dbeta, dS0 = torch.empty(B, H, L, **f), torch.empty(B, H, dk_, dv_, **f)
    need = int(_lib.efla_prefill_bwd_workspace_size(B, H, L, dk_, dv_))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(_lib.efla_prefill_bwd(_ptr(q), _ptr(k), _ptr(v), _dt(k), MODES[mode], _ptr(beta), _ptr(S0),
                                     _ptr(dO), _ptr(dSL), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbeta), _ptr(dS0),
                                     B, H, L, dk_, dv_, _ptr(workspace) if need else None,
                                     wbytes if need else 0, _stream(dev)),
               "efla_prefill_bwd")
    return dq, dk, dv, dbeta, dS0


def prefill_bwd_workspace_size(B: int, H: int, L: int, d: int) -> int:
    return int(_lib.efla_prefill_bwd_workspace_size(B, H, L, d, d))

