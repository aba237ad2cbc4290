"""Error measures and pass gates shared by the GPU parity tests.

Two measures, both against the fp64 oracle on the same input bits:

* normwise:    max_i |y_i - r_i| / max_i |r_i|.  The target's "max relative error"
  read normwise; its tolerances are 1e-5 for fp32 I/O and 2e-2 for bf16 I/O.
* elementwise: max_i |y_i - r_i| / max(|r_i|, 1e-3 rms(r)).  Reported beside it, so
  that an error confined to a region of small outputs is visible.

The gate takes both: normwise within the target tolerance, and every element within
rtol |r_i| + 1e-3 rms(r).  rtol follows from the arithmetic: a bf16 output is rounded
once (at most 2^-9 of its value), so 1e-2 leaves a factor of five for the fp32
arithmetic before it; fp32 outputs carry a few 1e-7 relative (approximate exp2 and
reciprocal, the decays' power chains), so 1e-5.
"""
import json
import os

import numpy as np
import torch

NORM_TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}
RTOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}
ATOL_FRAC = 1e-3
REPORT = os.environ.get("VIMSCAN_PARITY_REPORT")


def as_np(y):
    if torch.is_tensor(y):
        return y.detach().to("cpu", torch.float64).numpy()
    return np.asarray(y, dtype=np.float64)


def measures(y, ref):
    """normwise and elementwise errors of y against ref, and the largest ratio of an
    element's error to its gate allowance (filled in by gate())."""
    y, ref = as_np(y), as_np(ref)
    diff = np.abs(y - ref)
    if diff.size == 0:
        return dict(normwise=0.0, elementwise=0.0, rms=0.0)
    den = np.max(np.abs(ref))
    rms = float(np.sqrt(np.mean(ref * ref)))
    normwise = float(np.max(diff) / den) if den > 0 else float(np.max(diff))
    floor = max(1e-3 * rms, np.finfo(np.float64).tiny)
    elementwise = float(np.max(diff / np.maximum(np.abs(ref), floor)))
    return dict(normwise=normwise, elementwise=elementwise, rms=rms)


def gate(name, y, ref, dtype, *, norm_tol=None, rtol=None, atol_frac=ATOL_FRAC, elementwise=True):
    """Assert both gates (the elementwise one unless ``elementwise`` is False) and record
    the measures in $VIMSCAN_PARITY_REPORT when it is set.  Returns the measures."""
    yn, rn = as_np(y), as_np(ref)
    assert yn.shape == rn.shape, (name, yn.shape, rn.shape)
    assert np.all(np.isfinite(yn)), f"{name}: non-finite output"
    m = measures(yn, rn)
    norm_tol = NORM_TOL[dtype] if norm_tol is None else norm_tol
    rtol = RTOL[dtype] if rtol is None else rtol
    if yn.size:
        allow = rtol * np.abs(rn) + atol_frac * m["rms"]
        m["gate_ratio"] = float(np.max(np.abs(yn - rn) / np.maximum(allow, np.finfo(np.float64).tiny)))
    else:
        m["gate_ratio"] = 0.0
    if REPORT:
        with open(REPORT, "a") as f:
            f.write(json.dumps({"case": name, "dtype": str(dtype), **m}) + "\n")
    assert m["normwise"] <= norm_tol, f"{name}: normwise error {m['normwise']:.3e} > {norm_tol:.0e}"
    if elementwise:
        assert m["gate_ratio"] <= 1.0, (
            f"{name}: an element is off by {m['gate_ratio']:.2f}x its allowance "
            f"({rtol:.0e} |r| + {atol_frac:.0e} rms(r)); elementwise error {m['elementwise']:.3e}")
    return m
