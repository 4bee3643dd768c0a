"""Parity metrics shared by the GPU tests.

fp32 inputs : max_i |o_i - r_i| / max(|r_i|, rms(r))   <= 1e-4  (max relative error with an RMS floor
              so that elements near zero do not dominate)
bf16 inputs : max_i |o_i - r_i| / rms(r)                <= 2e-2  (fp32 accumulation on the GPU)
r is the fp64 oracle result on the identical stored inputs.

The bf16 bar is applied to the raw difference.  The exception is an output so heavy-tailed
that the exact result rounded to bf16 is itself further than 2e-2 of the RMS from the exact
value, so that no bf16 output could pass: the 3x3 conv layer (56x56, C = 64: max|o|/rms =
11.7, rounding alone 2.46e-2; `rounding_floor=True`) and the one-way chunked scans (80x80:
max|o|/rms = 8.5, rounding alone 2.15e-2; `rounding_floor="auto"`, which first checks that
the exact result's own rounding fails the bar).  There, half a bf16 ulp at max(|o_i|, |r_i|)
is taken off each difference before the bar, so that the bar measures the arithmetic beyond
the output's own rounding.  Both numbers are returned and printed.
"""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def _np(x):
    if hasattr(x, "detach"):
        return x.detach().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def half_ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def rounding_alone(ref):
    """max|bf16(r) - r| / rms(r): how far the exact result rounded to bf16 is from it."""
    r = np.asarray(ref, dtype=np.float64)
    rounded = torch.tensor(r, dtype=torch.float64).to(torch.bfloat16).double().numpy()
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    return float(np.max(np.abs(rounded - r), initial=0.0)) / rms if rms > 0 else 0.0


def err(gpu, ref, dtype, rounding_floor=False):
    """Returns (metric, raw): `metric` is what the bar applies to, `raw` = max|diff| / rms."""
    g = _np(gpu)
    r = np.asarray(ref, dtype=np.float64)
    if rounding_floor == "auto":
        rounding_floor = dtype == torch.bfloat16 and rounding_alone(r) > TOL[torch.bfloat16]
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    stored_bf16 = hasattr(gpu, "dtype") and gpu.dtype == torch.bfloat16
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    diff = np.abs(g - r)
    raw = float(np.max(diff, initial=0.0)) / rms if rms > 0 else float(np.max(diff, initial=0.0))
    if dtype == torch.float32:
        if rms == 0.0:
            return float(np.max(diff, initial=0.0)), raw
        return float(np.max(diff / np.maximum(np.abs(r), rms), initial=0.0)), raw
    if rounding_floor and stored_bf16:
        diff = np.maximum(diff - half_ulp_bf16(np.maximum(np.abs(g), np.abs(r))), 0.0)
    if rms == 0.0:
        return float(np.max(diff, initial=0.0)), raw
    return float(np.max(diff, initial=0.0)) / rms, raw


def assert_close(gpu, ref, dtype, what="", rounding_floor=False):
    e, raw = err(gpu, ref, dtype, rounding_floor=rounding_floor)
    print(f"{what}: metric {e:.3e} raw max|diff|/rms {raw:.3e}")
    assert e <= TOL[dtype], f"{what}: error {e:.3e} > {TOL[dtype]:.0e} (raw max|diff|/rms {raw:.3e})"
    return e
