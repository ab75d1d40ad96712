"""Shared helpers of the parity tests: tolerances and device transfer.

Tolerances (stated for the EFLA token mixer parity contract):
* fp32 inputs: max|x - ref| / max|ref| <= 1e-4 per output tensor (o, S_L);
* bf16 inputs with fp32 state: max|x - ref| <= 2e-2 * RMS(ref) per tensor.
``ref`` is always the fp64 oracle evaluated on the same (already rounded)
inputs.  These bars hold for fp32 outputs.  When the caller asks for a bf16
o, the rounding of each output element to bf16 (up to 2^-8 of |ref|) is
added on top: |x - ref| <= bar + 2^-8 |ref| elementwise ("bf16-out").
"""
import numpy as np
import torch

F32_REL = 1e-4
BF16_RMS = 2e-2


def np64(t):
    return t.detach().to("cpu").double().numpy() if hasattr(t, "detach") else np.asarray(t, np.float64)


def rel_max_err(x, ref):
    x, ref = np64(x), np64(ref)
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (den if den > 0 else 1.0))


def rms_err(x, ref):
    x, ref = np64(x), np64(ref)
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.abs(x - ref).max() / (rms if rms > 0 else 1.0))


def assert_close(x, ref, dtype, what="", out_bf16=False):
    """Apply the parity bar of ``dtype`` ("f32" or "bf16"); ``out_bf16`` adds
    the bf16 output-rounding term."""
    if out_bf16:
        xn, rn = np64(x), np64(ref)
        bar = (F32_REL * np.abs(rn).max()) if dtype == "f32" else BF16_RMS * np.sqrt(np.mean(rn ** 2))
        excess = np.abs(xn - rn) - (bar + 2.0 ** -8 * np.abs(rn))
        assert excess.max() <= 0, f"{what}: bf16-out bar exceeded by {excess.max():.3e}"
        return float(excess.max())
    if dtype == "f32":
        e = rel_max_err(x, ref)
        assert e <= F32_REL, f"{what}: max rel err {e:.3e} > {F32_REL}"
    else:
        e = rms_err(x, ref)
        assert e <= BF16_RMS, f"{what}: max err / RMS {e:.3e} > {BF16_RMS}"
    return e


def cuda(d):
    return {k: (v.cuda() if v is not None else None) for k, v in d.items()}
