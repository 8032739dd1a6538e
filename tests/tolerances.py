"""Parity tolerances, fixed in advance and never widened to make a test pass.

Scaled error err = |gpu - oracle| / (1 + |oracle|), element by element, with the
oracle run in fp64 on the same stored input bits:
  fp32 inputs:  y and states <= 1e-4,  gradients <= 1e-3
  bf16 / fp16 inputs with fp32 accumulation: everything <= 2e-2
"""
import numpy as np

TOL = {
    ("f32", "fwd"): 1e-4,
    ("f32", "grad"): 1e-3,
    ("bf16", "fwd"): 2e-2,
    ("bf16", "grad"): 2e-2,
    ("f16", "fwd"): 2e-2,
    ("f16", "grad"): 2e-2,
}


def assert_close(got, ref, tol, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert got.size > 0, f"{what}: nothing compared"
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref) / (1.0 + np.abs(ref))
    i = np.unravel_index(int(np.argmax(err)), err.shape)
    assert err.max() <= tol, (f"{what}: max scaled err {err.max():.3e} > {tol:.1e} at {i}: "
                              f"got {got[i]!r} ref {ref[i]!r}")
    return got.size
