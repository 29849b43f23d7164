"""Python binding of the C ABI in ``include/ssm_scan.h`` (ctypes, marshalling only).

Functions keep the C names (``ssm_scan_fwd``, ``ssm_scan_bwd``, ...) and take
torch CUDA tensors (or raw device addresses as ``int``, or ``None`` for NULL).
Every step of the scan runs in the CUDA library; nothing here computes.  The
library must have been built (``python -m selective_diagonal_state_b200.build``)
- there is no fallback: a missing library or a non-CUDA tensor raises.
"""
from __future__ import annotations

import ctypes
import os

from .synthetic import ScanShape

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm_scan.so")

SSM_OK = 0
STATUS = {0: "SSM_OK", -1: "SSM_ERR_ARG", -2: "SSM_ERR_UNSUPPORTED", -3: "SSM_ERR_ALIGN",
          -4: "SSM_ERR_CUDA", -5: "SSM_ERR_TIMEOUT", -6: "SSM_ERR_WORKSPACE"}
PASS_FWD, PASS_BWD, PASS_FWD_INFER = 0, 1, 2

EXPORTED = ["ssm_desc_set_contiguous", "ssm_scan_workspace_size", "ssm_scan_fwd",
            "ssm_scan_bwd", "ssm_scan_last_error", "ssm_scan_poll_device_error",
            "ssm_scan_abi_version", "ssm_scan_profile_start", "ssm_scan_profile_stop",
            "ssm_scan_bwd_noalloc", "ssm_scan_last_route", "ssm_scan_bwd_saved",
            "ssm_scan_step", "ssm_preact_fwd", "ssm_preact_bwd", "ssm_scan_set_wait_limit",
            "ssm_cp_tail_rows", "ssm_cp_segment_transition", "ssm_cp_state_combine",
            "ssm_cp_adjoint_combine", "ssm_cp_fill_tail", "ssm_cp_write_adjoint",
            "ssm_scan_fwd_gated", "ssm_gate_bwd"]
ROUTE_CHUNKED, ROUTE_RANGE_FALLBACK, ROUTE_RECURRENT, ROUTE_SSD, ROUTE_CHANNEL = 0, 1, 2, 3, 4
NOALLOC_SCRATCH_BYTES = 32 << 20


class SsmError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where} -> {STATUS.get(code, code)}: {msg}")
        self.code = code


class Desc(ctypes.Structure):
    """Mirror of ``ssm_desc_t``."""

    _fields_ = [
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
        ("headdim", ctypes.c_int64), ("ngroups", ctypes.c_int64),
        ("n_real", ctypes.c_int32), ("n_pairs", ctypes.c_int32),
        ("rank_in", ctypes.c_int32), ("rank_out", ctypes.c_int32),
        ("chunk", ctypes.c_int32), ("decay_mode", ctypes.c_int32),
        ("two_endpoint", ctypes.c_int32), ("dtype_io", ctypes.c_int32),
        ("stride_x", ctypes.c_int64 * 3), ("stride_y", ctypes.c_int64 * 3),
        ("stride_B", ctypes.c_int64 * 3), ("stride_C", ctypes.c_int64 * 3),
        ("stride_dt", ctypes.c_int64 * 3), ("stride_lambda", ctypes.c_int64 * 3),
        ("angle_mode", ctypes.c_int32), ("n_static", ctypes.c_int32),
        ("discretization", ctypes.c_int32), ("reserved_", ctypes.c_int32),
    ]


_lib = None
_vp = ctypes.c_void_p


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing: build it with "
                           "`python -m selective_diagonal_state_b200.build` (no CPU fallback)")
    lib = ctypes.CDLL(path)
    lib.ssm_desc_set_contiguous.argtypes = [ctypes.POINTER(Desc)]
    lib.ssm_desc_set_contiguous.restype = None
    lib.ssm_scan_workspace_size.argtypes = [ctypes.POINTER(Desc), ctypes.c_int]
    lib.ssm_scan_workspace_size.restype = ctypes.c_size_t
    lib.ssm_scan_fwd.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 14 + [ctypes.c_size_t, _vp]
    lib.ssm_scan_fwd.restype = ctypes.c_int
    lib.ssm_scan_bwd.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 22 + [ctypes.c_size_t, _vp]
    lib.ssm_scan_bwd.restype = ctypes.c_int
    lib.ssm_scan_bwd_noalloc.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 21 + [_vp]
    lib.ssm_scan_bwd_noalloc.restype = ctypes.c_int
    lib.ssm_scan_bwd_saved.argtypes = ([ctypes.POINTER(Desc)] + [_vp] * 22 +
                                       [ctypes.c_size_t, _vp, ctypes.c_size_t, _vp])
    lib.ssm_scan_bwd_saved.restype = ctypes.c_int
    lib.ssm_scan_step.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 12
    lib.ssm_scan_step.restype = ctypes.c_int
    lib.ssm_preact_fwd.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 6
    lib.ssm_preact_fwd.restype = ctypes.c_int
    lib.ssm_preact_bwd.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 9
    lib.ssm_preact_bwd.restype = ctypes.c_int
    lib.ssm_scan_fwd_gated.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 16 + [ctypes.c_size_t, _vp]
    lib.ssm_scan_fwd_gated.restype = ctypes.c_int
    lib.ssm_gate_bwd.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 6
    lib.ssm_gate_bwd.restype = ctypes.c_int
    lib.ssm_cp_tail_rows.argtypes = [ctypes.POINTER(Desc)]
    lib.ssm_cp_tail_rows.restype = ctypes.c_int
    lib.ssm_cp_segment_transition.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 7
    lib.ssm_cp_segment_transition.restype = ctypes.c_int
    lib.ssm_cp_state_combine.argtypes = ([ctypes.POINTER(Desc), ctypes.c_int, ctypes.c_int] +
                                         [_vp] * 9)
    lib.ssm_cp_state_combine.restype = ctypes.c_int
    lib.ssm_cp_adjoint_combine.argtypes = ([ctypes.POINTER(Desc), ctypes.c_int, ctypes.c_int] +
                                           [_vp] * 7)
    lib.ssm_cp_adjoint_combine.restype = ctypes.c_int
    lib.ssm_cp_fill_tail.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 8
    lib.ssm_cp_fill_tail.restype = ctypes.c_int
    lib.ssm_cp_write_adjoint.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 6
    lib.ssm_cp_write_adjoint.restype = ctypes.c_int
    lib.ssm_scan_last_error.argtypes = []
    lib.ssm_scan_last_error.restype = ctypes.c_char_p
    lib.ssm_scan_poll_device_error.argtypes = [_vp]
    lib.ssm_scan_poll_device_error.restype = ctypes.c_int
    lib.ssm_scan_abi_version.argtypes = []
    lib.ssm_scan_abi_version.restype = ctypes.c_int
    lib.ssm_scan_profile_start.argtypes = [ctypes.c_int]
    lib.ssm_scan_profile_start.restype = ctypes.c_int
    lib.ssm_scan_profile_stop.argtypes = [ctypes.c_char_p, ctypes.c_int,
                                          ctypes.POINTER(ctypes.c_int),
                                          ctypes.POINTER(ctypes.c_double), ctypes.c_int]
    lib.ssm_scan_profile_stop.restype = ctypes.c_int
    lib.ssm_scan_last_route.argtypes = [_vp]
    lib.ssm_scan_last_route.restype = ctypes.c_int
    lib.ssm_scan_set_wait_limit.argtypes = [ctypes.c_int64]
    lib.ssm_scan_set_wait_limit.restype = ctypes.c_int64
    _lib = lib
    return lib


def make_desc(shape: ScanShape) -> Desc:
    """Descriptor with dense strides for ``shape``."""
    d = Desc()
    d.batch, d.seqlen, d.nheads = shape.batch, shape.seqlen, shape.nheads
    d.headdim, d.ngroups = shape.headdim, shape.ngroups
    d.n_real, d.n_pairs = shape.n_real, shape.n_pairs
    d.rank_in, d.rank_out = shape.rank_in, shape.rank_out
    d.chunk, d.decay_mode = shape.chunk, shape.decay_mode
    d.two_endpoint, d.dtype_io = shape.two_endpoint, shape.dtype_io
    d.angle_mode, d.n_static = shape.angle_mode, shape.n_static
    d.discretization = shape.discretization
    load_library().ssm_desc_set_contiguous(ctypes.byref(d))
    return d


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not getattr(t, "is_cuda", False):
        raise ValueError("ssm_scan: every tensor must live on a CUDA device (no CPU path)")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != SSM_OK:
        msg = load_library().ssm_scan_last_error().decode(errors="replace")
        raise SsmError(rc, where, msg)


def ssm_scan_workspace_size(desc: Desc, pass_: int) -> int:
    return int(load_library().ssm_scan_workspace_size(ctypes.byref(desc), pass_))


def ssm_scan_fwd(desc: Desc, x, dt, A_log, theta, B, C, D, lam, h0, prev_write, y, hT=None,
                 last_write=None, workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_scan_fwd(ctypes.byref(desc), *[_ptr(t) for t in (
        x, dt, A_log, theta, B, C, D, lam, h0, prev_write, y, hT, last_write, workspace)],
        workspace_bytes, _stream(stream))
    _check(rc, "ssm_scan_fwd")


def ssm_scan_step(desc: Desc, x, dt, A_log, theta, B, C, D, lam, h, w, y, stream=None) -> None:
    """One recurrent step; ``h`` and ``w`` (fp32 state and previous write) are
    updated in place."""
    lib = load_library()
    rc = lib.ssm_scan_step(ctypes.byref(desc), *[_ptr(t) for t in (
        x, dt, A_log, theta, B, C, D, lam, h, w, y)], _stream(stream))
    _check(rc, "ssm_scan_step")


def ssm_scan_fwd_gated(desc: Desc, x, dt, A_log, theta, B, C, D, lam, h0, prev_write, z,
                       y_gated, y_pre=None, hT=None, last_write=None, workspace=None,
                       workspace_bytes: int = 0, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_scan_fwd_gated(ctypes.byref(desc), *[_ptr(t) for t in (
        x, dt, A_log, theta, B, C, D, lam, h0, prev_write, z, y_gated, y_pre, hT, last_write,
        workspace)], workspace_bytes, _stream(stream))
    _check(rc, "ssm_scan_fwd_gated")


def ssm_gate_bwd(desc: Desc, z, y_pre, dy_gated, dy, dz, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_gate_bwd(ctypes.byref(desc), *[_ptr(t) for t in (z, y_pre, dy_gated, dy, dz)],
                          _stream(stream))
    _check(rc, "ssm_gate_bwd")


def ssm_cp_tail_rows(desc: Desc) -> int:
    n = int(load_library().ssm_cp_tail_rows(ctypes.byref(desc)))
    _check(SSM_OK if n >= 0 else -1, "ssm_cp_tail_rows")
    return n


def ssm_cp_segment_transition(desc: Desc, dt, A_log, theta, lam, phi, beta0, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_cp_segment_transition(ctypes.byref(desc), *[_ptr(t) for t in (
        dt, A_log, theta, lam, phi, beta0)], _stream(stream))
    _check(rc, "ssm_cp_segment_transition")


def ssm_cp_state_combine(desc: Desc, nseg: int, seg: int, hT_all, wT_all, phi_all, beta0_all,
                         h0, w0, h_in, w_in, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_cp_state_combine(ctypes.byref(desc), nseg, seg, *[_ptr(t) for t in (
        hT_all, wT_all, phi_all, beta0_all, h0, w0, h_in, w_in)], _stream(stream))
    _check(rc, "ssm_cp_state_combine")


def ssm_cp_adjoint_combine(desc: Desc, nseg: int, seg: int, dh0_all, phi_all, beta0_all, dhT,
                           dh_end, dw_end, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_cp_adjoint_combine(ctypes.byref(desc), nseg, seg, *[_ptr(t) for t in (
        dh0_all, phi_all, beta0_all, dhT, dh_end, dw_end)], _stream(stream))
    _check(rc, "ssm_cp_adjoint_combine")


def ssm_cp_fill_tail(desc: Desc, x, dt, B, C, lam, dy, dh_end, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_cp_fill_tail(ctypes.byref(desc), *[_ptr(t) for t in (
        x, dt, B, C, lam, dy, dh_end)], _stream(stream))
    _check(rc, "ssm_cp_fill_tail")


def ssm_cp_write_adjoint(desc: Desc, x, B, dw_end, dx, dB, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_cp_write_adjoint(ctypes.byref(desc), *[_ptr(t) for t in (
        x, B, dw_end, dx, dB)], _stream(stream))
    _check(rc, "ssm_cp_write_adjoint")


def ssm_preact_fwd(desc: Desc, z, dt_bias, lam_logit, dt, lam, stream=None) -> None:
    """dt = softplus(z + dt_bias[h]); lam = sigmoid(lam_logit) (two-endpoint)."""
    lib = load_library()
    rc = lib.ssm_preact_fwd(ctypes.byref(desc), *[_ptr(t) for t in (
        z, dt_bias, lam_logit, dt, lam)], _stream(stream))
    _check(rc, "ssm_preact_fwd")


def ssm_preact_bwd(desc: Desc, z, dt_bias, lam_logit, ddt, dlam, dz, ddt_bias=None,
                   dlam_logit=None, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_preact_bwd(ctypes.byref(desc), *[_ptr(t) for t in (
        z, dt_bias, lam_logit, ddt, dlam, dz, ddt_bias, dlam_logit)], _stream(stream))
    _check(rc, "ssm_preact_bwd")


def ssm_scan_bwd(desc: Desc, x, dt, A_log, theta, B, C, D, lam, h0, prev_write, dy, dx, ddt,
                 dA_log, dtheta, dB, dC, dD, dlam=None, dh0=None, dprev_write=None,
                 workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    lib = load_library()
    rc = lib.ssm_scan_bwd(ctypes.byref(desc), *[_ptr(t) for t in (
        x, dt, A_log, theta, B, C, D, lam, h0, prev_write, dy, dx, ddt, dA_log, dtheta, dB, dC,
        dD, dlam, dh0, dprev_write, workspace)], workspace_bytes, _stream(stream))
    _check(rc, "ssm_scan_bwd")


def ssm_scan_bwd_saved(desc: Desc, x, dt, A_log, theta, B, C, D, lam, h0, prev_write, dy, dx,
                       ddt, dA_log, dtheta, dB, dC, dD, dlam=None, dh0=None, dprev_write=None,
                       fwd_workspace=None, fwd_workspace_bytes: int = 0, workspace=None,
                       workspace_bytes: int = 0, stream=None) -> None:
    """Backward reading the chunk states from the workspace of a preceding
    forward on the same inputs."""
    lib = load_library()
    rc = lib.ssm_scan_bwd_saved(ctypes.byref(desc), *[_ptr(t) for t in (
        x, dt, A_log, theta, B, C, D, lam, h0, prev_write, dy, dx, ddt, dA_log, dtheta, dB, dC,
        dD, dlam, dh0, dprev_write, fwd_workspace)], fwd_workspace_bytes, _ptr(workspace),
        workspace_bytes, _stream(stream))
    _check(rc, "ssm_scan_bwd_saved")


def ssm_scan_bwd_noalloc(desc: Desc, x, dt, A_log, theta, B, C, D, lam, h0, prev_write, dy, dx,
                         ddt, dA_log, dtheta, dB, dC, dD, dlam=None, dh0=None, dprev_write=None,
                         stream=None) -> None:
    """Backward without a workspace argument: the library's fixed device
    scratch is used instead (for callers that cannot allocate device memory)."""
    lib = load_library()
    rc = lib.ssm_scan_bwd_noalloc(ctypes.byref(desc), *[_ptr(t) for t in (
        x, dt, A_log, theta, B, C, D, lam, h0, prev_write, dy, dx, ddt, dA_log, dtheta, dB, dC,
        dD, dlam, dh0, dprev_write)], _stream(stream))
    _check(rc, "ssm_scan_bwd_noalloc")


def ssm_scan_poll_device_error(stream=None) -> None:
    _check(load_library().ssm_scan_poll_device_error(_stream(stream)),
           "ssm_scan_poll_device_error")


def ssm_scan_set_wait_limit(polls: int) -> int:
    """Polls of a carry counter before a chained kernel's wait gives up (0: every
    such wait gives up); returns the previous limit."""
    rc = int(load_library().ssm_scan_set_wait_limit(int(polls)))
    if rc < 0:
        _check(rc, "ssm_scan_set_wait_limit")
    return rc


def ssm_scan_abi_version() -> int:
    return int(load_library().ssm_scan_abi_version())


def ssm_scan_last_route(stream=None) -> int:
    """Route of the last scan call on this thread (ROUTE_*); synchronises the stream."""
    rc = int(load_library().ssm_scan_last_route(_stream(stream)))
    if rc < 0:
        _check(rc, "ssm_scan_last_route")
    return rc


def ssm_scan_profile_start(max_launches: int) -> None:
    _check(load_library().ssm_scan_profile_start(max_launches), "ssm_scan_profile_start")


def ssm_scan_profile_stop(max_kernels: int = 32) -> dict:
    """Close the timing session; returns {kernel: (launches, total_ms)}."""
    lib = load_library()
    name_len = 48
    names = ctypes.create_string_buffer(name_len * max_kernels)
    counts = (ctypes.c_int * max_kernels)()
    tot = (ctypes.c_double * max_kernels)()
    n = lib.ssm_scan_profile_stop(names, name_len, counts, tot, max_kernels)
    if n < 0:
        _check(n, "ssm_scan_profile_stop")
    out = {}
    for i in range(n):
        nm = names.raw[i * name_len:(i + 1) * name_len].split(b"\0", 1)[0].decode()
        out[nm] = (int(counts[i]), float(tot[i]))
    return out
