"""Helpers shared by the tests (comparison metric; no method arithmetic)."""
import numpy as np

BF16_TOL = 2e-2   # max relative error, bf16 inputs with fp32 accumulation
FP32_TOL = 1e-4   # max relative error, fp32 mode


def slice_rel_err(got, ref, unit_axes):
    """max over (b, h) slices of max|got - ref| / max|ref| within the slice.

    unit_axes: the axes of the (b, h) unit in the array (e.g. (0, 2) for
    [B, T, H, dv], (0, 1) for [B, H, dv, dk])."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if got.size == 0:
        return 0.0
    other = tuple(a for a in range(ref.ndim) if a not in unit_axes)
    num = np.max(np.abs(got - ref), axis=other)
    den = np.max(np.abs(ref), axis=other)
    den = np.where(den > 0, den, 1.0)
    if not np.all(np.isfinite(got)):
        return float("inf")
    return float(np.max(num / den))
