"""Comparison metrics and tolerances shared by the parity tests.

max_rel = max|got - ref| / max|ref|   (per output tensor)
rel_l2  = ||got - ref||_2 / ||ref||_2
Bars: fp32 inputs max_rel <= 1e-4; bf16 inputs max_rel <= 2e-2 and
rel_l2 <= 5e-3 (fp32 accumulation, bf16 operands and bf16 y).
"""
import numpy as np

TOL = {"f32": {"max_rel": 1e-4, "rel_l2": 1e-4}, "bf16": {"max_rel": 2e-2, "rel_l2": 5e-3}}


def metrics(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return {"max_rel": 0.0, "rel_l2": 0.0}
    err = got - ref
    scale = np.abs(ref).max()
    l2 = np.sqrt((ref ** 2).sum())
    return {"max_rel": float(np.abs(err).max() / scale) if scale > 0 else float(np.abs(err).max()),
            "rel_l2": float(np.sqrt((err ** 2).sum()) / l2) if l2 > 0 else float(np.sqrt((err ** 2).sum()))}


def assert_close(got, ref, dtype, what=""):
    m = metrics(got, ref)
    tol = TOL[dtype]
    assert np.isfinite(np.asarray(got, dtype=np.float64)).all(), f"{what}: non-finite output"
    assert m["max_rel"] <= tol["max_rel"] and m["rel_l2"] <= tol["rel_l2"], f"{what}: {m} vs {tol}"
    return m
