"""Shared helpers of the GPU parity tests (comparison metrics, tolerances).

Tolerances of the scan, per output tensor:

* fp32 inputs/outputs: rel-L2 <= 1e-5.
* bf16 inputs/outputs with fp32 state: rel-L2 <= 2e-2 and a per-element
  max-abs bound that starts from the stated 5e-2:
    - outputs stored as bf16 (y, dx, ddt, dB, dC, dlambda):
      |gpu - ref| <= 5e-2 + 2^-8 |ref|.  Storing a value of magnitude m in
      bf16 alone moves it by up to m 2^-9 (round to nearest, 8 stored
      mantissa bits), so a flat 5e-2 cannot hold above |ref| = 25.6; the
      relative term allows twice that storage rounding and no more.
    - outputs stored as fp32 (hT, last_write, dA_log, dtheta, dD, dh0,
      dprev_write): |gpu - ref| <= 5e-2 flat, no relative slack, unless the
      caller passes a derived bound for a long parameter reduction (see
      ``param_bound``).
The largest error of every compared tensor is recorded in ``report`` (and in
the module-level ``LAST``) whether or not the check passes.
"""
import numpy as np

TOL = {0: dict(rel_l2=1e-5, max_abs=None), 1: dict(rel_l2=2e-2, max_abs=5e-2)}
BF16_REL = 2.0 ** -8
FP32_STORED = {"hT", "last_write", "dA_log", "dtheta", "dD", "dh0", "dprev_write"}
LAST = {}


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def param_bound(n_terms, ref):
    """Per-element bound of a parameter gradient that sums ``n_terms`` token
    contributions (batch x length of one head) in fp32 from operands carried
    with about 16 mantissa bits (bf16 hi + lo pairs) and bf16-rounded inputs.

    Each contribution is exact up to a relative 2^-16 of its own size, and the
    errors of different tokens are independent, so the error of the sum grows
    like sqrt(n_terms) times the typical term, i.e. |sum| 2^-16 sqrt(n) at
    worst when the terms do not cancel.  Returns max(5e-2, that) per element."""
    ref = np.abs(np.asarray(ref, dtype=np.float64))
    return np.maximum(5e-2, ref * 2.0 ** -16 * np.sqrt(float(n_terms)))


def compare(name, got, ref, dtype_io, report=None, bound=None):
    """Assert the tolerance of ``name`` (see the module docstring); ``bound``
    overrides the per-element max-abs bound (array or scalar) for a derived
    case.  Returns (rel-L2, max-abs)."""
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
    LAST[name] = (rel, mabs)
    if report is not None:
        report[name] = (rel, mabs)
    assert rel <= tol["rel_l2"], f"{name}: rel-L2 {rel:.3e} > {tol['rel_l2']}"
    if tol["max_abs"] is not None and got.size:
        if bound is not None:
            lim = np.broadcast_to(np.asarray(bound, dtype=np.float64), err.shape)
        elif name in FP32_STORED:
            lim = np.full(err.shape, tol["max_abs"])
        else:
            lim = tol["max_abs"] + BF16_REL * np.abs(ref)
        ratio = err / lim
        i = int(np.argmax(ratio))
        assert ratio.flat[i] <= 1.0, (
            f"{name}: |err| {err.flat[i]:.3e} at |ref| {abs(ref.flat[i]):.3e} exceeds "
            f"the bound {lim.flat[i]:.3e} (max-abs over the tensor {mabs:.3e})")
    return rel, mabs
