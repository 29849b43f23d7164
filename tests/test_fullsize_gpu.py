"""Parity at the full HybridMamba size (8 x 8192 tokens, 32 heads, 64 real +
32 rotation pairs, two-endpoint, bf16 I/O), in the launch configuration the
benchmark times: a training forward into its workspace, then the backward that
reads it.  The oracle recomputes sampled heads (every batch row, the whole
sequence; B and C are per head, so a head is an independent problem) and every
output of those heads is compared element by element, including the per-head
parameter gradients."""
import numpy as np
import pytest

import oracle
from selective_diagonal_state_b200 import abi, scan
from selective_diagonal_state_b200 import synthetic as S
from tests.parity_util import compare, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SAMPLED_HEADS = (0, 13, 31)


@pytest.fixture(scope="module")
def full_run():
    from selective_diagonal_state_b200 import build
    build.build()
    abi.load_library()
    shape = S.WORKLOADS["hybridmamba"]
    assert shape.ngroups == shape.nheads
    inp = S.make_inputs(shape, seed=4)
    dev = scan.to_device(shape, inp)
    wsf = scan.alloc_workspace(shape, abi.PASS_FWD)
    y, hT, wT = scan.scan_forward(shape, dev, workspace=wsf)
    assert abi.ssm_scan_last_route() == abi.ROUTE_CHUNKED
    g = scan.scan_backward(shape, dev, saved=wsf)
    assert abi.ssm_scan_last_route() == abi.ROUTE_CHUNKED
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    out = dict(y=to_np(y), hT=to_np(hT), wT=to_np(wT), dx=to_np(g.dx), ddt=to_np(g.ddt),
               dB=to_np(g.dBm), dC=to_np(g.dCm), dlam=to_np(g.dlam), dA_log=to_np(g.dA_log),
               dtheta=to_np(g.dtheta), dD=to_np(g.dD))
    del dev, wsf, y, hT, wT, g
    torch.cuda.empty_cache()
    return shape, inp, out


@pytest.mark.parametrize("h", SAMPLED_HEADS)
def test_sampled_head_at_full_size(full_run, h):
    shape, inp, out = full_run
    sub = shape.replace(nheads=1, ngroups=1)
    hs = slice(h, h + 1)
    si = {k: inp[k][:, :, hs] for k in ("x", "dt", "lam", "Bm", "Cm", "dy")}
    si.update(A_log=inp["A_log"][hs], theta=inp["theta"][hs], D=inp["D"][hs])
    ref = oracle.scan_fwd(sub, si)
    grad = oracle.scan_bwd(sub, si, si["dy"])
    dt = shape.dtype_io
    compare("y", out["y"][:, :, hs], ref["y"], dt)
    compare("hT", out["hT"][:, hs], ref["hT"], dt)
    compare("last_write", out["wT"][:, hs], ref["wT"], dt)
    compare("dx", out["dx"][:, :, hs], grad["dx"], dt)
    compare("ddt", out["ddt"][:, :, hs], grad["ddt"], dt)
    compare("dB", out["dB"][:, :, hs], grad["dBm"], dt)
    compare("dC", out["dC"][:, :, hs], grad["dCm"], dt)
    compare("dlambda", out["dlam"][:, :, hs], grad["dlam"], dt)
    compare("dA_log", out["dA_log"][hs], grad["dA_log"], dt)
    compare("dtheta", out["dtheta"][hs], grad["dtheta"], dt)
    compare("dD", out["dD"][hs], grad["dD"], dt)
