"""Shared helpers of the GPU parity tests: tolerances and comparisons.

Tolerances (stated with the method's accuracy targets):
  * final state:  max|S - S_ref| <= 2e-3 * max|S_ref|
  * outputs / hidden, bf16 inputs: max|x - x_ref| / max|x_ref| <= 1e-2
  * outputs and state, fp32-input mode: <= 1e-4 in the same normwise sense
The relative error is normwise over a whole tensor (the max abs error divided
by the max abs reference value): an elementwise relative error is unbounded
near zero, and the GPU rounds intermediates to bf16 by design.
"""
import numpy as np

STATE_TOL = 2e-3
OUT_TOL_BF16 = 1e-2
TOL_FP32 = 1e-4


def to_np(t):
    return t.detach().float().cpu().double().numpy() if hasattr(t, "detach") else np.asarray(t)


def normwise_err(got, ref):
    got = to_np(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in GPU output"
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    err = np.max(np.abs(got - ref)) if ref.size else 0.0
    return err / scale if scale > 0 else err


def assert_close(got, ref, tol, what=""):
    e = normwise_err(got, ref)
    assert e <= tol, f"{what}: normwise error {e:.3e} > {tol:.1e}"
    return e
