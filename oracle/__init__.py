"""fp64 CPU oracle for the selective diagonal scan -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it.

``oracle_scan.c`` holds the arithmetic (a plain sequential recurrence and its
hand-written reverse mode, see the header comment there for the passages it
follows).  This module only builds it with gcc and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle_scan.c")
_LIB = os.path.join(_HERE, "liboracle_scan.so")
_lib = None


class _Desc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_long), ("seqlen", ctypes.c_long), ("nheads", ctypes.c_long),
        ("headdim", ctypes.c_long), ("ngroups", ctypes.c_long),
        ("n_real", ctypes.c_int), ("n_pairs", ctypes.c_int),
        ("rank_in", ctypes.c_int), ("rank_out", ctypes.c_int),
        ("per_coord_decay", ctypes.c_int), ("two_endpoint", ctypes.c_int),
        ("angle_per_token", ctypes.c_int),
        ("n_static", ctypes.c_int),
        ("zoh", ctypes.c_int),
    ]


def build(force: bool = False, extra_flags=()) -> str:
    """Compile the oracle with gcc (-O2, OpenMP over independent (b, h) units)."""
    out = _LIB
    if extra_flags:
        tag = "_".join(f.strip("-").replace("=", "") for f in extra_flags)
        out = os.path.join(_HERE, f"liboracle_scan_{tag}.so")
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", *extra_flags, _SRC,
               "-o", out, "-lm"]
        subprocess.check_call(cmd)
    return out


def _load(path=None):
    global _lib
    if path is not None:
        return ctypes.CDLL(path)
    if _lib is None:
        _lib = ctypes.CDLL(build())
    return _lib


def _desc(shape) -> _Desc:
    return _Desc(shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.ngroups,
                 shape.n_real, shape.n_pairs, shape.rank_in, shape.rank_out,
                 1 if shape.decay_mode == 1 else 0, shape.two_endpoint,
                 1 if getattr(shape, "angle_mode", 0) == 1 else 0, getattr(shape, "n_static", 0),
                 1 if getattr(shape, "discretization", 0) == 1 else 0)


def _p(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def scan_fwd(shape, inp: dict, lib_path=None) -> dict:
    """Run the oracle forward.  ``inp`` holds the arrays of ``synthetic.make_inputs``."""
    lib = _load(lib_path)
    s = shape
    d = _desc(s)
    a = {k: _f64(inp.get(k)) for k in ("x", "dt", "A_log", "theta", "Bm", "Cm", "D", "lam",
                                        "h0", "w0")}
    if a["theta"] is None or a["theta"].size == 0:
        a["theta"] = np.zeros(max(1, s.nheads * s.n_pairs))
    if a["lam"] is None:
        a["lam"] = np.ones((s.batch, s.seqlen, s.nheads))
    y = np.zeros((s.batch, s.seqlen, s.nheads, s.rank_out, s.headdim))
    hT = np.zeros((s.batch, s.nheads, s.nstate, s.headdim))
    wT = np.zeros_like(hT)
    lib.oracle_scan_fwd.restype = ctypes.c_int
    rc = lib.oracle_scan_fwd(ctypes.byref(d), _p(a["x"]), _p(a["dt"]), _p(a["A_log"]),
                             _p(a["theta"]), _p(a["Bm"]), _p(a["Cm"]), _p(a["D"]), _p(a["lam"]),
                             _p(a["h0"]), _p(a["w0"]), _p(y), _p(hT), _p(wT))
    if rc != 0:
        raise RuntimeError(f"oracle_scan_fwd failed: {rc}")
    return {"y": y, "hT": hT, "wT": wT}


def scan_bwd(shape, inp: dict, dy, lib_path=None) -> dict:
    """Run the oracle backward for upstream gradient ``dy`` (shape of ``y``)."""
    lib = _load(lib_path)
    s = shape
    d = _desc(s)
    a = {k: _f64(inp.get(k)) for k in ("x", "dt", "A_log", "theta", "Bm", "Cm", "D", "lam",
                                        "h0", "w0")}
    if a["theta"] is None or a["theta"].size == 0:
        a["theta"] = np.zeros(max(1, s.nheads * s.n_pairs))
    if a["lam"] is None:
        a["lam"] = np.ones((s.batch, s.seqlen, s.nheads))
    dy = _f64(dy)
    out = {
        "dx": np.zeros_like(a["x"]), "ddt": np.zeros_like(a["dt"]),
        "dA_log": np.zeros_like(a["A_log"]),
        "dtheta": (np.zeros((s.batch, s.seqlen, s.nheads, s.n_pairs))
                   if getattr(s, "angle_mode", 0) == 1 else np.zeros((s.nheads, s.n_pairs))),
        "dBm": np.zeros_like(a["Bm"]), "dCm": np.zeros_like(a["Cm"]),
        "dD": np.zeros_like(a["D"]), "dlam": np.zeros((s.batch, s.seqlen, s.nheads)),
        "dh0": np.zeros((s.batch, s.nheads, s.nstate, s.headdim)),
        "dw0": np.zeros((s.batch, s.nheads, s.nstate, s.headdim)),
    }
    dth = out["dtheta"] if s.n_pairs > 0 else np.zeros(1)
    lib.oracle_scan_bwd.restype = ctypes.c_int
    rc = lib.oracle_scan_bwd(ctypes.byref(d), _p(a["x"]), _p(a["dt"]), _p(a["A_log"]),
                             _p(a["theta"]), _p(a["Bm"]), _p(a["Cm"]), _p(a["D"]), _p(a["lam"]),
                             _p(a["h0"]), _p(a["w0"]), _p(dy), _p(out["dx"]), _p(out["ddt"]),
                             _p(out["dA_log"]), _p(dth), _p(out["dBm"]), _p(out["dCm"]),
                             _p(out["dD"]), _p(out["dlam"]), _p(out["dh0"]), _p(out["dw0"]))
    if rc != 0:
        raise RuntimeError(f"oracle_scan_bwd failed: {rc}")
    if s.n_pairs > 0:
        out["dtheta"] = dth
    return out


# ---------------------------------------------------------------------------
# Pre-activations of dt and lambda (fp64).  The pages give the log-uniform
# initialisation of the step ("State Space Models", robocikowo.com, the entries
# on the discretisation step); the positivity maps are the reading the
# workloads use: dt = softplus(z + dt_bias[h]), lambda = sigmoid(logit).
# Parity pinned by closed forms and central differences in
# tests/test_preact_pins.py.
# ---------------------------------------------------------------------------
def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    # 1 / (1 + e^-x), written with e^-|x| so that neither side loses relative precision
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def preact_fwd(z, dt_bias, lam_logit=None):
    """dt[b,t,h] = softplus(z[b,t,h] + dt_bias[h]); lam = sigmoid(lam_logit)."""
    z = np.asarray(z, dtype=np.float64)
    dt = _softplus(z + np.asarray(dt_bias, dtype=np.float64)[None, None, :])
    lam = None if lam_logit is None else _sigmoid(np.asarray(lam_logit, dtype=np.float64))
    return dt, lam


def preact_bwd(z, dt_bias, lam_logit, ddt, dlam=None):
    """Chain rule through preact_fwd: (dz, ddt_bias, dlam_logit)."""
    x = np.asarray(z, dtype=np.float64) + np.asarray(dt_bias, dtype=np.float64)[None, None, :]
    dz = np.asarray(ddt, dtype=np.float64) * _sigmoid(x)
    dbias = dz.sum(axis=(0, 1))
    dlogit = None
    if lam_logit is not None and dlam is not None:
        lam = _sigmoid(np.asarray(lam_logit, dtype=np.float64))
        dlogit = np.asarray(dlam, dtype=np.float64) * lam * (1.0 - lam)
    return dz, dbias, dlogit


# ---- output gate of the mixer ------------------------------------------------------
# The pages' fused kernel merges the state update with the gating and the output
# projection of the mixer ("Diagonal Equivalence in State Space Models", kongchang.com:
# the kernel-performance paragraph).  Reading (the gate's form is not given there): the
# Mamba-style output gate y_g = y * silu(z), z of y's shape, silu(z) = z sigmoid(z).
def gate_fwd(y, z):
    """y_g = y * silu(z), elementwise."""
    y = np.asarray(y, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    return y * z * _sigmoid(z)


def gate_bwd(y, z, dyg):
    """Chain rule through gate_fwd: (dy, dz) for the upstream gradient dyg."""
    y = np.asarray(y, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    g = np.asarray(dyg, dtype=np.float64)
    s = _sigmoid(z)
    dy = g * z * s
    dz = g * y * s * (1.0 + z * (1.0 - s))
    return dy, dz

