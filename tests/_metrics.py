"""Parity metric for yhat (shared by the GPU tests and the smoke check).

err = max over rows i of ||y_i - ref_i||_inf / max(||ref_i||_inf, 1e-6): the maximum relative
error per output row.  Per-element relative error is unstable where yhat is near zero, so
each row is normalised by its largest entry."""
import numpy as np


def row_rel_err(y, ref):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    num = np.abs(y - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-6)
    return float((num / den).max())


TOL_F32 = 1e-4   # fp32 path
TOL_BF16 = 2e-2  # bf16 inputs, fp32 accumulation
