"""Helpers shared by the GPU parity tests (no arithmetic of the method here)."""
from __future__ import annotations

import numpy as np

# The acceptance rule for fp32 results against the fp64 oracle:
#     |out_gpu - out_ref| <= REL * twin + ABS   elementwise,
# where twin is the oracle's magnitude companion (the same expression over
# absolute values), which bounds the rounding error of any fp32 evaluation.
REL = 1e-5
ABS = 1e-30


def assert_close(gpu, ref, twin, name="", rel=REL, abs_=ABS):
    gpu = np.asarray(gpu, dtype=np.float64).reshape(np.shape(ref))
    ref = np.asarray(ref, dtype=np.float64)
    twin = np.asarray(twin, dtype=np.float64).reshape(np.shape(ref))
    err = np.abs(gpu - ref)
    bound = rel * twin + abs_
    bad = ~(err <= bound)  # NaN counts as bad
    if bad.any():
        idx = np.flatnonzero(bad.reshape(-1))[:5]
        worst = np.nanmax(err / np.maximum(bound, 1e-300))
        raise AssertionError(
            f"{name}: {int(bad.sum())} of {bad.size} elements out of tolerance; worst err/bound {worst:.3g}; "
            f"first at {idx.tolist()}: gpu={gpu.reshape(-1)[idx]}, ref={ref.reshape(-1)[idx]}, "
            f"twin={twin.reshape(-1)[idx]}")
    return float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0
