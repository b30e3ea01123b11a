"""Helpers shared by the GPU parity tests (not a test module)."""

import numpy as np

# Tolerances of the method's parity contract: max elementwise relative error
# |g - r| / (|r| + rms(r)) against the float64 oracle.
TOL_F32 = 1e-4     # float32 I/O, float32 arithmetic
TOL_BF16 = 2e-2    # bfloat16 I/O, float32 accumulation and state


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rms = np.sqrt(np.mean(ref * ref)) + 1e-300
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + rms)))


def norm_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / (np.linalg.norm(ref) + 1e-300))


def assert_close(got, ref, tol, what=""):
    e = rel_err(got, ref)
    n = norm_err(got, ref)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite output"
    assert e <= tol, f"{what}: max rel err {e:.3g} > {tol} (normwise {n:.3g})"
    return e


def host(t):
    return t.float().cpu().numpy()
