"""The C-ABI library loads and exports every call include/efla.h declares,
and its synchronous argument validation rejects bad calls before touching
a GPU (no compute calls here; these run on a CPU-only machine)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "efla.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(efla_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import delta_rule_linear_03_b200 as efla
    return efla._lib, efla


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("efla_gate", "efla_chunk_fwd", "efla_decode_step"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so, efla = lib
    for name in declared_functions():
        assert hasattr(so, name), f"libefla.so does not export {name}"


def test_status_strings_and_version(lib):
    so, efla = lib
    assert efla.version() >= 100
    for code, name in efla.STATUS.items():
        assert so.efla_status_string(code).decode().startswith(name)


A = ctypes.c_void_p(0x10000)  # aligned fake device addresses: never dereferenced
A2 = ctypes.c_void_p(0x20000)
A3 = ctypes.c_void_p(0x30000)
A4 = ctypes.c_void_p(0x40000)
A5 = ctypes.c_void_p(0x50000)
A6 = ctypes.c_void_p(0x60000)


def test_validation_rejects_before_launch(lib):
    so, efla = lib
    F32, BF16 = 0, 1
    # bad dtype / mode
    assert so.efla_chunk_fwd(A, A2, A3, 7, 0, A4, None, A5, 0, None, 1, 1, 64, 128, 128, None, 0, None) == 3
    assert so.efla_chunk_fwd(A, A2, A3, F32, 9, A4, None, A5, 0, None, 1, 1, 64, 128, 128, None, 0, None) == 3
    assert so.efla_chunk_fwd(A, A2, A3, F32, 0, A4, None, A5, 5, None, 1, 1, 64, 128, 128, None, 0, None) == 3
    # unsupported head sizes
    assert so.efla_chunk_fwd(A, A2, A3, F32, 0, A4, None, A5, 0, None, 1, 1, 64, 48, 48, None, 0, None) == 5
    assert so.efla_chunk_fwd(A, A2, A3, F32, 0, A4, None, A5, 0, None, 1, 1, 64, 128, 64, None, 0, None) == 5
    assert so.efla_decode_step(A, A2, A3, F32, 0, A4, A5, A6, 0, 1, 1, 256, 256, None) == 5
    # negative sizes
    assert so.efla_chunk_fwd(A, A2, A3, F32, 0, A4, None, A5, 0, None, -1, 1, 64, 128, 128, None, 0, None) == 2
    assert so.efla_gate(A, F32, 0, A2, A3, None, 1, 1, -5, 128, None) == 2
    # NULL required pointers
    assert so.efla_chunk_fwd(None, A2, A3, F32, 0, A4, None, A5, 0, None, 1, 1, 64, 128, 128, None, 0, None) == 1
    assert so.efla_decode_step(A, A2, A3, BF16, 0, A4, None, A6, 0, 1, 1, 128, 128, None) == 1
    assert so.efla_gate(None, F32, 0, A2, A3, None, 1, 1, 5, 128, None) == 1
    # misaligned pointers
    bad = ctypes.c_void_p(0x10004)
    assert so.efla_chunk_fwd(bad, A2, A3, F32, 0, A4, None, A5, 0, None, 1, 1, 64, 128, 128, None, 0, None) == 4
    assert so.efla_decode_step(A, A2, A3, F32, 0, A4, bad, A6, 0, 1, 1, 128, 128, None) == 4
    # aliasing: o on top of q
    assert so.efla_chunk_fwd(A, A2, A3, F32, 0, A4, None, A, 0, None, 1, 1, 64, 128, 128, None, 0, None) == 9
    # workspace required for the fp32 path and absent
    need = so.efla_chunk_fwd_workspace_size(F32, 1, 1, 64, 128, 128)
    assert need > 0
    assert so.efla_chunk_fwd(A, A2, A3, F32, 0, A4, None, A5, 0, None, 1, 1, 64, 128, 128, None, 0, None) == 8
    # empty problems are accepted without any launch
    assert so.efla_chunk_fwd(None, None, None, F32, 0, None, None, None, 0, None, 0, 4, 64, 128, 128, None, 0,
                             None) == 0
    assert so.efla_decode_step(None, None, None, F32, 0, None, None, None, 0, 3, 0, 64, 64, None) == 0
    assert so.efla_gate(None, F32, 0, None, None, None, 2, 2, 0, 32, None) == 0
    # L = 0 without S_L: nothing to do
    assert so.efla_chunk_fwd(None, None, None, BF16, 0, None, None, None, 0, None, 2, 2, 0, 64, 64, None, 0,
                             None) == 0


def test_workspace_size_is_pure_and_scales(lib):
    so, _ = lib
    a = so.efla_chunk_fwd_workspace_size(0, 2, 16, 8192, 128, 128)
    b = so.efla_chunk_fwd_workspace_size(0, 2, 16, 8192, 128, 128)
    assert a == b and a > 0
    assert so.efla_chunk_fwd_workspace_size(0, 4, 16, 8192, 128, 128) == 2 * a
    assert so.efla_chunk_fwd_workspace_size(0, 2, 16, 8192, 48, 48) == 0
    assert so.efla_chunk_fwd_workspace_size(0, 0, 16, 8192, 128, 128) == 0


def test_bf16_workspace_includes_segment_states(lib):
    # bf16 d=128 path: one 56 KB image per (b, h, chunk); with too few heads to
    # fill the GPU the prefill is segmented (P segments) and adds 3P - 5 fp32
    # states of d x d per (b, h).  Without a GPU the plan assumes 148 SMs.
    so, _ = lib
    img = 7 * 8192
    st = 128 * 128 * 4
    # 64 heads, 32 chunks: a single pass
    assert so.efla_chunk_fwd_workspace_size(1, 8, 8, 2048, 128, 128) == 64 * 32 * img
    # 16 heads, 1024 chunks: P = 5 (pass A needs 2 CTAs per segment and head: 2 * 16 * 4 = 128)
    assert so.efla_chunk_fwd_workspace_size(1, 1, 16, 65536, 128, 128) == 16 * 1024 * img + 10 * 16 * st
    # 2 heads, 128 chunks: P = 8 (16 chunks per segment)
    assert so.efla_chunk_fwd_workspace_size(1, 1, 2, 8192, 128, 128) == 2 * 128 * img + 19 * 2 * st
    # too few chunks per segment: a single pass
    assert so.efla_chunk_fwd_workspace_size(1, 1, 2, 2048, 128, 128) == 2 * 32 * img


def test_state_affine_validation(lib):
    import ctypes
    so, _ = lib
    p = ctypes.c_void_p(16)
    so.efla_state_affine.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 3 + [ctypes.c_void_p]
    assert so.efla_state_affine(p, p, p, ctypes.c_void_p(1 << 20), 1, 1, 48, None) == 5  # UNSUPPORTED
    assert so.efla_state_affine(None, p, p, p, 1, 1, 64, None) == 1                      # NULL
    assert so.efla_state_affine(p, p, p, p, -1, 1, 64, None) == 2                        # SHAPE
    assert so.efla_state_affine(p, p, p, p, 0, 1, 64, None) == 0                         # empty: OK
    assert so.efla_state_affine(p, p, p, ctypes.c_void_p(20), 1, 1, 64, None) == 4       # ALIGN
    assert so.efla_state_affine(p, p, p, p, 1, 1, 64, None) == 9                         # ALIAS


def test_prefill_bwd_validation(lib):
    import ctypes
    so, _ = lib
    P = ctypes.c_void_p
    so.efla_prefill_bwd.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int] + [P] * 9 + [ctypes.c_int] * 5 + \
        [P, ctypes.c_size_t, P]
    so.efla_prefill_bwd_workspace_size.restype = ctypes.c_size_t
    ptrs = [P(16 * (i + 1) << 20) for i in range(12)]  # distinct, aligned, far apart
    q, k, v, beta, S0, dO, dSL, dq, dk, dv, db, dS = ptrs
    ws = P(64 << 30)

    def call(**kw):
        a = dict(q=q, k=k, v=v, dt=0, mode=0, beta=beta, S0=S0, dO=dO, dSL=dSL, dq=dq, dk=dk, dv=dv, db=db,
                 dS=dS, B=1, H=2, L=8, dk_=64, dv_=64, ws=ws, wsb=1 << 30)
        a.update(kw)
        return so.efla_prefill_bwd(a["q"], a["k"], a["v"], a["dt"], a["mode"], a["beta"], a["S0"], a["dO"],
                                   a["dSL"], a["dq"], a["dk"], a["dv"], a["db"], a["dS"], a["B"], a["H"], a["L"],
                                   a["dk_"], a["dv_"], a["ws"], a["wsb"], None)

    assert call(dq=None) == 1                      # NULL
    assert call(dk_=48, dv_=48) == 5               # UNSUPPORTED head size
    assert call(dt=7) == 3                         # DTYPE
    assert call(L=-1) == 2                         # SHAPE
    assert call(dq=P((16 << 20) + 4)) == 4         # ALIGN
    assert call(dq=q) == 9                         # ALIAS (output over an input)
    assert call(ws=None) == 8                      # WORKSPACE missing
    assert call(wsb=16) == 8                       # WORKSPACE too small
    assert call(B=0) == 0                          # empty batch: nothing to do
    assert so.efla_prefill_bwd_workspace_size(1, 2, 8, 64, 64) == 2 * 8 * (64 + 5) * 4
