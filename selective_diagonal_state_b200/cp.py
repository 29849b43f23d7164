"""Sequence sharding (context parallelism) of the scan.

A sequence of length L is split into ``nseg`` consecutive segments, one per
rank.  Each rank scans its own segment with the library's kernels; the
segments are joined exactly through per-segment boundary values (the
composition rule and the C calls are documented with ``ssm_cp_*`` in
``include/ssm_scan.h``):

forward   1. scan the segment from a zero state -> its local end state and last
             write, and its whole transition Phi (``ssm_cp_segment_transition``);
          2. all-gather those over the ranks (the one exchange of the forward);
          3. ``ssm_cp_state_combine`` -> the state and left endpoint entering
             this segment; scan the segment again from them -> exact y, hT.
backward  1. the segment's backward with no end adjoint -> its local dh0;
          2. all-gather the local dh0 (the one exchange of the backward);
          3. ``ssm_cp_adjoint_combine`` -> the adjoint entering the segment's
             end (and its last write's); the backward again with that end
             adjoint (fed through ``ssm_cp_fill_tail``'s trailing rows) and
             ``ssm_cp_write_adjoint`` -> exact gradients of the segment's
             tokens; the per-head parameter gradients are summed over ranks.

Every step runs in the CUDA library; this module holds the buffers, the
order of the calls and the collectives.  The forward's step 1 writes no y
(a state-only forward); the exact forward keeps its chunk states, and both
backwards (step 1 for the local dh0, step 3 the exact one) read them.  A readout-only correction (instead of the second forward scan) and an
adjoint-only first backward are the cheaper forms left for later.  Per-token rotation angles and static rows are not sharded
(the trailing rows cannot pass them through unchanged).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import abi, scan
from .synthetic import ANGLE_PER_TOKEN, ScanShape


def _torch():
    import torch
    return torch


def segment_bounds(seqlen: int, nseg: int, seg: int) -> tuple:
    """Token range [start, stop) of segment `seg` (the first seqlen % nseg
    segments take one token more)."""
    if nseg < 1 or not 0 <= seg < nseg:
        raise ValueError("bad segment index")
    base, extra = divmod(seqlen, nseg)
    start = seg * base + min(seg, extra)
    return start, start + base + (1 if seg < extra else 0)


@dataclasses.dataclass
class Boundary:
    """What a segment publishes: local end state, last write, transition, beta_0."""
    hT: object
    wT: object
    phi: object
    beta0: object


class SegmentScan:
    """Device buffers of one segment: token tensors hold ``tail`` trailing rows
    after the segment's own ``seqlen`` (``ssm_cp_tail_rows``), through which the
    backward receives the adjoint of the segment's end state."""

    def __init__(self, shape: ScanShape, device="cuda"):
        if shape.angle_mode == ANGLE_PER_TOKEN and shape.n_pairs:
            raise ValueError("sequence sharding: per-token rotation angles are not supported")
        if shape.n_static:
            raise ValueError("sequence sharding: static rows are not supported")
        torch = _torch()
        self.shape = shape
        self.tail = abi.ssm_cp_tail_rows(abi.make_desc(shape))
        self.ext = shape.replace(seqlen=shape.seqlen + self.tail)
        s, e = self.ext, shape
        io = scan.io_dtype(s)
        z = lambda *sz, dt=io: torch.zeros(sz, dtype=dt, device=device)  # noqa: E731
        f32 = torch.float32
        self.dev = scan.DeviceInputs(
            x=z(s.batch, s.seqlen, s.nheads, s.rank_in, s.headdim),
            dt=z(s.batch, s.seqlen, s.nheads),
            A_log=z(s.nheads, s.n_decay, dt=f32),
            theta=z(s.nheads, s.n_pairs, dt=f32) if s.n_pairs else None,
            Bm=z(s.batch, s.seqlen, s.ngroups, s.rank_in, s.nstate),
            Cm=z(s.batch, s.seqlen, s.ngroups, s.rank_out, s.nstate),
            D=z(s.nheads, dt=f32),
            lam=z(s.batch, s.seqlen, s.nheads) if s.two_endpoint else None,
            dy=z(s.batch, s.seqlen, s.nheads, s.rank_out, s.headdim))
        self.out = scan.alloc_fwd(s, device)            # y over the extended rows
        self.grads = scan.alloc_bwd(s, device)
        st = (e.batch, e.nheads, e.nstate, e.headdim)
        self.h_in, self.w_in = z(*st, dt=f32), z(*st, dt=f32)
        self.dh_end, self.dw_end = z(*st, dt=f32), z(*st, dt=f32)
        nmode = e.n_real + e.n_pairs
        self.bnd = Boundary(hT=z(*st, dt=f32), wT=z(*st, dt=f32),
                            phi=z(e.batch, e.nheads, nmode, 2, dt=f32),
                            beta0=z(e.batch, e.nheads, dt=f32))
        self.dh0_loc = z(*st, dt=f32)
        # the extended buffers' descriptor, and the segment's own (same strides)
        self.desc_ext = abi.make_desc(self.ext)
        self.desc = abi.Desc.from_buffer_copy(self.desc_ext)
        self.desc.seqlen = shape.seqlen
        # the state-only forward of step 1 (y not written) takes the training size
        self.ws_s = scan.alloc_workspace(shape, abi.PASS_FWD, device, self.desc)
        # the exact forward runs over the extended rows and keeps its chunk states,
        # which both backwards read
        self.ws_f = scan.alloc_workspace(self.ext, abi.PASS_FWD, device, self.desc_ext)
        self.ws_b = scan.alloc_workspace(self.ext, abi.PASS_BWD, device, self.desc_ext)

    # ---- inputs ---------------------------------------------------------------------
    def load(self, inp: dict, start: int, stop: int) -> None:
        """Copy tokens [start, stop) of a whole-sequence input dict (synthetic
        layout, host arrays) and its parameters into the segment's buffers."""
        torch = _torch()
        d, L = self.dev, self.shape.seqlen
        assert stop - start == L
        io = scan.io_dtype(self.shape)

        def put(dst, a):
            dst[:, :L].copy_(torch.from_numpy(np.ascontiguousarray(a[:, start:stop])).to(io))

        put(d.x, inp["x"])
        put(d.dt, inp["dt"])
        put(d.Bm, inp["Bm"])
        put(d.Cm, inp["Cm"])
        if d.lam is not None:
            put(d.lam, inp["lam"])
        if "dy" in inp:
            put(d.dy, inp["dy"])
        d.A_log.copy_(torch.from_numpy(inp["A_log"]))
        if d.theta is not None:
            d.theta.copy_(torch.from_numpy(inp["theta"]))
        d.D.copy_(torch.from_numpy(inp["D"]))

    # ---- forward ----------------------------------------------------------------------
    def forward_local(self) -> Boundary:
        """Step 1: the segment's end state from a zero state (a state-only forward:
        no y), and its transition."""
        d, b = self.dev, self.bnd
        abi.ssm_scan_fwd(self.desc, d.x, d.dt, d.A_log, d.theta, d.Bm, d.Cm, d.D, d.lam, None,
                         None, None, b.hT, b.wT, self.ws_s[0], self.ws_s[1])
        abi.ssm_cp_segment_transition(self.desc, d.dt, d.A_log, d.theta, d.lam, b.phi, b.beta0)
        return b

    def forward_exact(self, nseg, seg, gathered: Boundary, h0=None, w0=None):
        """Step 3: the entering state from the gathered boundaries, then the
        segment from it, over the extended rows (the trailing rows pass the state
        through unchanged and change no y of the segment's tokens), keeping the
        chunk states for the backward.  Returns (y of the segment's tokens, hT,
        last write); the last write is the segment's own, from step 1."""
        d = self.dev
        abi.ssm_cp_state_combine(self.desc, nseg, seg, gathered.hT, gathered.wT, gathered.phi,
                                 gathered.beta0, h0, w0, self.h_in, self.w_in)
        # the trailing rows' inputs as the backward reads them (its end adjoint only
        # changes their dy, which the forward does not read)
        abi.ssm_cp_fill_tail(self.desc, d.x, d.dt, d.Bm, d.Cm, d.lam, d.dy, None)
        y, hT, wT = self.out
        abi.ssm_scan_fwd(self.desc_ext, d.x, d.dt, d.A_log, d.theta, d.Bm, d.Cm, d.D, d.lam,
                         self.h_in, self.w_in, y, hT, wT, self.ws_f[0], self.ws_f[1])
        return y[:, :self.shape.seqlen], hT, self.bnd.wT

    # ---- backward ---------------------------------------------------------------------
    def _backward(self, dh_end):
        # reads the chunk states the exact forward kept (same inputs, entering
        # state and trailing rows; only the trailing rows' dy differ)
        d, g = self.dev, self.grads
        # the trailing rows' other inputs were written before the exact forward
        abi.ssm_cp_fill_tail(self.desc, None, None, None, None, None, d.dy, dh_end)
        args = (self.desc_ext, d.x, d.dt, d.A_log, d.theta, d.Bm, d.Cm, d.D, d.lam, self.h_in,
                self.w_in, d.dy, g.dx, g.ddt, g.dA_log, g.dtheta, g.dBm, g.dCm, g.dD, g.dlam,
                g.dh0, g.dw0)
        if self.ws_f[1]:
            abi.ssm_scan_bwd_saved(*args, self.ws_f[0], self.ws_f[1], self.ws_b[0], self.ws_b[1])
        else:   # a forward that keeps nothing (the recurrent kernels)
            abi.ssm_scan_bwd(*args, self.ws_b[0], self.ws_b[1])

    def backward_local(self):
        """Step 1: the backward with no end adjoint -> the local dh0 (after
        ``forward_exact``, whose kept chunk states it reads)."""
        self._backward(None)
        self.dh0_loc.copy_(self.grads.dh0)
        return self.dh0_loc

    def backward_exact(self, nseg, seg, dh0_all, gathered: Boundary, dhT=None) -> scan.Grads:
        """Step 3: the end adjoint from the gathered local dh0 of the later
        segments, then the backward with it.  The returned token gradients hold
        the extended rows; the segment's own are the first ``shape.seqlen``."""
        abi.ssm_cp_adjoint_combine(self.desc, nseg, seg, dh0_all, gathered.phi, gathered.beta0,
                                   dhT, self.dh_end, self.dw_end)
        self._backward(self.dh_end)
        d, g = self.dev, self.grads
        abi.ssm_cp_write_adjoint(self.desc, d.x, d.Bm, self.dw_end, g.dx, g.dBm)
        return g


def stack_boundaries(bnds) -> Boundary:
    """The gathered form ("_all" arrays) of per-segment boundaries, in segment order."""
    torch = _torch()
    return Boundary(*(torch.stack([getattr(b, f) for b in bnds]).contiguous()
                      for f in ("hT", "wT", "phi", "beta0")))


def run_sharded(segs, h0=None, w0=None, dhT=None, backward=True):
    """All segments of one sequence processed one after another on one device:
    the sharded algorithm with the all-gathers done by stacking (every rank's
    kernels run separately; none waits on another).  Returns per-segment
    forward outputs and gradients."""
    torch = _torch()
    nseg = len(segs)
    bnds = [s.forward_local() for s in segs]
    gathered = stack_boundaries(bnds)
    fwd = [s.forward_exact(nseg, k, gathered, h0, w0) for k, s in enumerate(segs)]
    if not backward:
        return fwd, None
    dh0_all = torch.stack([s.backward_local() for s in segs]).contiguous()
    grads = [s.backward_exact(nseg, k, dh0_all, gathered, dhT) for k, s in enumerate(segs)]
    return fwd, grads


def all_gather_stacked(t, world, group=None):
    """[world, *t.shape] tensor of every rank's `t`, in rank order (one all-gather)."""
    torch = _torch()
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts).contiguous()


def train_step(seg: SegmentScan, rank: int, world: int, group=None, h0=None, w0=None,
               dhT=None):
    """One sharded forward + backward on `world` ranks (this rank holds
    segment `rank`): two all-gathers of boundary values and the all-reduce of
    the per-head parameter gradients.  Returns (y, hT, last write, grads) of this
    rank's segment."""
    from . import dist as sdist
    b = seg.forward_local()
    gathered = Boundary(*(all_gather_stacked(getattr(b, f), world, group)
                          for f in ("hT", "wT", "phi", "beta0")))
    y, hT, wT = seg.forward_exact(world, rank, gathered, h0, w0)
    dh0_all = all_gather_stacked(seg.backward_local(), world, group)
    g = seg.backward_exact(world, rank, dh0_all, gathered, dhT)
    sdist.allreduce_param_grads((g.dA_log, g.dtheta, g.dD), group)
    return y, hT, wT, g


__all__ = ["Boundary", "SegmentScan", "segment_bounds", "stack_boundaries", "run_sharded",
           "all_gather_stacked", "train_step"]
