"""Torch-facing helpers around the C ABI: device buffers in, device buffers out.

PyTorch is used only for device memory and streams.  These helpers move
arrays to the GPU, allocate outputs and workspace with ``torch.empty`` and call
``ssm_scan_fwd`` / ``ssm_scan_bwd``; every arithmetic step runs in the CUDA
library.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import abi
from .synthetic import ANGLE_PER_TOKEN, DTYPE_BF16, ScanShape


def _torch():
    import torch
    return torch


def io_dtype(shape: ScanShape):
    torch = _torch()
    return torch.bfloat16 if shape.dtype_io == DTYPE_BF16 else torch.float32


@dataclasses.dataclass
class DeviceInputs:
    """Inputs of one scan on the GPU (dtype_io tensors, fp32 parameters)."""

    x: object
    dt: object
    A_log: object
    theta: object
    Bm: object
    Cm: object
    D: object
    lam: object
    dy: object = None
    h0: object = None
    w0: object = None


def to_device(shape: ScanShape, inp: dict, device="cuda", pin=False) -> DeviceInputs:
    """Copy host arrays (``synthetic.make_inputs`` layout) to the device."""
    torch = _torch()
    dt_io = io_dtype(shape)

    def io(a):
        if a is None:
            return None
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dt_io)
        return t.to(device, non_blocking=pin)

    def f32(a):
        if a is None:
            return None
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)

    theta = inp.get("theta")
    return DeviceInputs(
        x=io(inp["x"]), dt=io(inp["dt"]), A_log=f32(inp["A_log"]),
        theta=f32(theta) if theta is not None and theta.size else None,
        Bm=io(inp["Bm"]), Cm=io(inp["Cm"]), D=f32(inp["D"]),
        lam=io(inp["lam"]) if shape.two_endpoint else None,
        dy=io(inp.get("dy")), h0=f32(inp.get("h0")), w0=f32(inp.get("w0")))


def alloc_fwd(shape: ScanShape, device="cuda"):
    torch = _torch()
    s = shape
    y = torch.empty((s.batch, s.seqlen, s.nheads, s.rank_out, s.headdim), dtype=io_dtype(s),
                    device=device)
    hT = torch.empty((s.batch, s.nheads, s.nstate, s.headdim), dtype=torch.float32, device=device)
    wT = torch.empty_like(hT)
    return y, hT, wT


def scan_forward(shape: ScanShape, dev: DeviceInputs, out=None, desc=None, stream=None,
                 workspace=None):
    """Run ``ssm_scan_fwd``; returns (y, hT, last_write).  ``workspace`` is a
    (tensor, bytes) pair from ``alloc_workspace(shape, PASS_FWD)``; allocated
    here when not given."""
    desc = desc or abi.make_desc(shape)
    y, hT, wT = out if out is not None else alloc_fwd(shape, dev.x.device)
    ws, nbytes = workspace if workspace is not None else alloc_workspace(
        shape, abi.PASS_FWD, dev.x.device, desc)
    abi.ssm_scan_fwd(desc, dev.x, dev.dt, dev.A_log, dev.theta, dev.Bm, dev.Cm, dev.D, dev.lam,
                     dev.h0, dev.w0, y, hT, wT, ws, nbytes, stream)
    return y, hT, wT


@dataclasses.dataclass
class Grads:
    dx: object
    ddt: object
    dA_log: object
    dtheta: object
    dBm: object
    dCm: object
    dD: object
    dlam: object
    dh0: object
    dw0: object


def alloc_bwd(shape: ScanShape, device="cuda"):
    torch = _torch()
    s = shape
    io = io_dtype(s)
    e = lambda *sz, dt=io: torch.empty(sz, dtype=dt, device=device)  # noqa: E731
    f = torch.float32
    g = Grads(
        dx=e(s.batch, s.seqlen, s.nheads, s.rank_in, s.headdim),
        ddt=e(s.batch, s.seqlen, s.nheads),
        dA_log=e(s.nheads, s.n_decay, dt=f),
        dtheta=(None if not s.n_pairs else
                e(s.batch, s.seqlen, s.nheads, s.n_pairs, dt=f) if s.angle_mode == ANGLE_PER_TOKEN
                else e(s.nheads, s.n_pairs, dt=f)),
        dBm=e(s.batch, s.seqlen, s.ngroups, s.rank_in, s.nstate),
        dCm=e(s.batch, s.seqlen, s.ngroups, s.rank_out, s.nstate),
        dD=e(s.nheads, dt=f),
        dlam=e(s.batch, s.seqlen, s.nheads) if s.two_endpoint else None,
        dh0=e(s.batch, s.nheads, s.nstate, s.headdim, dt=f),
        dw0=e(s.batch, s.nheads, s.nstate, s.headdim, dt=f))
    return g


def alloc_workspace(shape: ScanShape, pass_: int, device="cuda", desc=None):
    torch = _torch()
    desc = desc or abi.make_desc(shape)
    n = abi.ssm_scan_workspace_size(desc, pass_)
    if n == 0:
        return None, 0
    return torch.empty(n, dtype=torch.uint8, device=device), n


def scan_backward(shape: ScanShape, dev: DeviceInputs, grads=None, workspace=None, desc=None,
                  stream=None, saved=None) -> Grads:
    """Run ``ssm_scan_bwd`` for ``dev.dy``; returns the gradient buffers.  With
    ``saved`` = the (tensor, bytes) forward workspace of a preceding
    ``scan_forward`` on the same inputs, ``ssm_scan_bwd_saved`` reuses its
    chunk states."""
    desc = desc or abi.make_desc(shape)
    g = grads or alloc_bwd(shape, dev.x.device)
    ws, nbytes = workspace if workspace is not None else alloc_workspace(
        shape, abi.PASS_BWD, dev.x.device, desc)
    args = (desc, dev.x, dev.dt, dev.A_log, dev.theta, dev.Bm, dev.Cm, dev.D, dev.lam, dev.h0,
            dev.w0, dev.dy, g.dx, g.ddt, g.dA_log, g.dtheta, g.dBm, g.dCm, g.dD, g.dlam, g.dh0,
            g.dw0)
    if saved is not None and saved[0] is not None:
        abi.ssm_scan_bwd_saved(*args, saved[0], saved[1], ws, nbytes, stream)
    else:
        abi.ssm_scan_bwd(*args, ws, nbytes, stream)
    return g
