"""Shared parity helpers for the GPU tests: tolerances and error reports.

Tolerances (bf16 inputs, fp32 accumulation, compared with the fp64 oracle):
max |err| <= 1e-2 and mean |err| <= 1e-3 on O, dQ, dK, dV; max |err| <= 1e-3
on LSE. Pattern expansion and block iteration are compared bit for bit.
"""

import numpy as np

MAX_TOL = 1e-2
MEAN_TOL = 1e-3
LSE_TOL = 1e-3


def report(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    err = np.abs(got - ref)
    return {
        "name": name,
        "max": float(err.max()) if err.size else 0.0,
        "mean": float(err.mean()) if err.size else 0.0,
        "n": int(err.size),
        "n_ref_ge4": int((np.abs(ref) >= 4).sum()),
        "nonfinite": int((~np.isfinite(got)).sum()),
    }


def assert_close(name, got, ref, max_tol=MAX_TOL, mean_tol=MEAN_TOL):
    r = report(name, got, ref)
    assert r["nonfinite"] == 0, r
    assert r["max"] <= max_tol and r["mean"] <= mean_tol, r
    return r


def assert_lse(name, got, ref, tol=LSE_TOL):
    r = report(name, got, ref)
    assert r["nonfinite"] == 0, r
    assert r["max"] <= tol, r
    return r
