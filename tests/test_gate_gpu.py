"""The mixer's output gate on the GPU: the gated forward (fused into the
per-coordinate tensor-core epilogue, an elementwise pass after the other
chains) and the gate's backward, against the oracle's scan and gate."""
import numpy as np
import pytest

import oracle
from selective_diagonal_state_b200 import abi, scan
from selective_diagonal_state_b200 import synthetic as S
from tests.parity_util import compare, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from selective_diagonal_state_b200 import build
    build.build()
    abi.load_library()


def _z(shape, seed):
    g = np.random.default_rng(seed)
    z = g.standard_normal((shape.batch, shape.seqlen, shape.nheads, shape.rank_out,
                           shape.headdim)).astype(np.float32)
    return S.round_bf16(z) if shape.dtype_io == S.DTYPE_BF16 else z


CASES = {
    "chunked (fused epilogue)": ("hybridmamba", dict(batch=2, nheads=4, ngroups=4, seqlen=150),
                                 abi.ROUTE_CHUNKED),
    "scalar-decay": ("ssd_mimo_r4", dict(batch=1, nheads=2, ngroups=2, seqlen=100), abi.ROUTE_SSD),
    "channel scan": ("mamba1_siso", dict(batch=2, nheads=64, seqlen=70), abi.ROUTE_CHANNEL),
    "recurrent fp32": ("tiny_hybrid_fp32", dict(seqlen=40), abi.ROUTE_RECURRENT),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("keep_pre", [True, False])
def test_gated_forward_and_gate_backward(case, keep_pre):
    name, kw, route = CASES[case]
    shape = S.WORKLOADS[name].replace(**kw)
    inp = S.make_inputs(shape, seed=41, with_state=True)
    z = _z(shape, 42)
    dev = scan.to_device(shape, inp)
    io = scan.io_dtype(shape)
    zd = torch.from_numpy(z).to(io).cuda()
    yg, hT, wT = scan.alloc_fwd(shape)
    ypre = torch.empty_like(yg) if keep_pre else None
    desc = abi.make_desc(shape)
    ws, nb = scan.alloc_workspace(shape, abi.PASS_FWD_INFER, desc=desc)
    abi.ssm_scan_fwd_gated(desc, dev.x, dev.dt, dev.A_log, dev.theta, dev.Bm, dev.Cm, dev.D,
                           dev.lam, dev.h0, dev.w0, zd, yg, ypre, hT, wT, ws, nb)
    assert abi.ssm_scan_last_route() == route
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    ref = oracle.scan_fwd(shape, inp)
    dt = shape.dtype_io
    compare("y_gated", to_np(yg), oracle.gate_fwd(ref["y"], z), dt)
    compare("hT", to_np(hT), ref["hT"], dt)
    if not keep_pre:
        return
    compare("y_pre", to_np(ypre), ref["y"], dt)
    g = np.random.default_rng(43).standard_normal(z.shape).astype(np.float32)
    if dt == S.DTYPE_BF16:
        g = S.round_bf16(g)
    gd = torch.from_numpy(g).to(io).cuda()
    dy, dz = torch.empty_like(gd), torch.empty_like(gd)
    abi.ssm_gate_bwd(desc, zd, ypre, gd, dy, dz)
    torch.cuda.synchronize()
    rdy, rdz = oracle.gate_bwd(ref["y"], z, g)
    compare("dy", to_np(dy), rdy, dt)
    compare("dz", to_np(dz), rdz, dt)


def test_gate_on_the_range_fallback():
    """A step too large for the tensor-core fold sends the call to the recurrent
    kernels behind the device-side gate; the gate pass runs on that chain only."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, seqlen=130)
    inp = S.make_inputs(shape, seed=44)
    inp["dt"] = S.round_bf16(inp["dt"] * np.float32(200.0))
    z = _z(shape, 45)
    dev = scan.to_device(shape, inp)
    zd = torch.from_numpy(z).to(scan.io_dtype(shape)).cuda()
    yg, hT, wT = scan.alloc_fwd(shape)
    ypre = torch.empty_like(yg)
    desc = abi.make_desc(shape)
    ws, nb = scan.alloc_workspace(shape, abi.PASS_FWD_INFER, desc=desc)
    abi.ssm_scan_fwd_gated(desc, dev.x, dev.dt, dev.A_log, dev.theta, dev.Bm, dev.Cm, dev.D,
                           dev.lam, None, None, zd, yg, ypre, hT, wT, ws, nb)
    assert abi.ssm_scan_last_route() == abi.ROUTE_RANGE_FALLBACK
    torch.cuda.synchronize()
    ref = oracle.scan_fwd(shape, inp)
    compare("y_gated", to_np(yg), oracle.gate_fwd(ref["y"], z), shape.dtype_io)
    compare("y_pre", to_np(ypre), ref["y"], shape.dtype_io)
