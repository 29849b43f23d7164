"""Shared helpers of the GPU parity tests (comparison metrics, tolerances)."""
import numpy as np

# Tolerances of the scan (per output tensor):
#   fp32 inputs/outputs:            rel-L2 <= 1e-5
#   bf16 inputs/outputs, fp32 state: rel-L2 <= 2e-2 and max-abs <= 5e-2
# The max-abs bound holds for values of unit scale and relatively above it:
# |gpu_i - ref_i| <= 5e-2 * max(1, |ref_i|) for every element, because bf16
# storage alone rounds a value of magnitude m by up to m * 2^-9 (a gradient
# of 17 already carries a rounding error of 0.06).
TOL = {0: dict(rel_l2=1e-5, max_abs=None), 1: dict(rel_l2=2e-2, max_abs=5e-2)}


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare(name, got, ref, dtype_io, report=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    tol = TOL[dtype_io]
    num = np.linalg.norm((got - ref).ravel())
    den = np.linalg.norm(ref.ravel())
    rel = num / den if den > 0 else num
    err = np.abs(got - ref)
    mabs = float(err.max()) if got.size else 0.0
    if report is not None:
        report[name] = (rel, mabs)
    assert rel <= tol["rel_l2"], f"{name}: rel-L2 {rel:.3e} > {tol['rel_l2']}"
    if tol["max_abs"] is not None and got.size:
        scaled = err / np.maximum(1.0, np.abs(ref))
        i = int(np.argmax(scaled))
        assert scaled.flat[i] <= tol["max_abs"], (
            f"{name}: |err| {err.flat[i]:.3e} at |ref| {abs(ref.flat[i]):.3e} exceeds "
            f"{tol['max_abs']} * max(1, |ref|)")
    return rel, mabs
