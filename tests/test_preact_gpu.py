"""GPU parity of the pre-activations (ssm_preact_fwd / ssm_preact_bwd) against
the oracle, and of the composed path z -> dt -> scan."""
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
    assert torch.cuda.is_available()


def _raw(shape, seed):
    """z ~ N(0, variance 0.5), dt_bias from a log-uniform dt0, logits ~ N(0, 1)."""
    g = np.random.default_rng(seed)
    B, L, H = shape.batch, shape.seqlen, shape.nheads
    dt0 = np.exp(g.uniform(np.log(1e-3), np.log(1e-1), size=H))
    bias = np.log(np.expm1(dt0)).astype(np.float32)
    z = (g.standard_normal((B, L, H)) * np.sqrt(0.5)).astype(np.float32)
    logit = g.standard_normal((B, L, H)).astype(np.float32)
    if shape.dtype_io == S.DTYPE_BF16:
        z, logit = S.round_bf16(z), S.round_bf16(logit)
    return z, bias, logit


def _dev(a, shape):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(scan.io_dtype(shape)).cuda()


@pytest.mark.parametrize("name,heads", [("tiny_hybrid_fp32", 0), ("hybridmamba", 4),
                                        ("mamba1_siso", 96), ("hybridmamba", 3),
                                        ("tiny_hybrid_fp32", 5)])
def test_preact_forward_and_backward(name, heads):
    """Both pre-activation passes against the oracle: dense layouts with an even
    head count take two heads per thread, odd head counts one element per thread."""
    shape = S.WORKLOADS[name].replace(batch=2, seqlen=37)
    if heads:
        shape = shape.replace(nheads=heads, ngroups=heads if name != "mamba1_siso" else 1)
    z, bias, logit = _raw(shape, 5)
    desc = abi.make_desc(shape)
    zd, ld = _dev(z, shape), _dev(logit, shape)
    bd = torch.from_numpy(bias).cuda()
    dt = torch.empty_like(zd)
    lam = torch.empty_like(ld)
    two = bool(shape.two_endpoint)
    abi.ssm_preact_fwd(desc, zd, bd, ld if two else None, dt, lam if two else None)
    rdt, rlam = oracle.preact_fwd(z, bias, logit if two else None)
    compare("dt", to_np(dt), rdt, shape.dtype_io)
    if two:
        compare("lambda", to_np(lam), rlam, shape.dtype_io)
    g = np.random.default_rng(6)
    ddt = g.standard_normal(z.shape).astype(np.float32)
    dlam = g.standard_normal(z.shape).astype(np.float32)
    if shape.dtype_io == S.DTYPE_BF16:
        ddt, dlam = S.round_bf16(ddt), S.round_bf16(dlam)
    dz = torch.empty_like(zd)
    dlg = torch.empty_like(ld)
    dbias = torch.empty(shape.nheads, dtype=torch.float32, device="cuda")
    abi.ssm_preact_bwd(desc, zd, bd, ld if two else None, _dev(ddt, shape),
                       _dev(dlam, shape) if two else None, dz, dbias, dlg if two else None)
    torch.cuda.synchronize()
    rdz, rdb, rdl = oracle.preact_bwd(z, bias, logit, ddt, dlam)
    compare("dz", to_np(dz), rdz, shape.dtype_io)
    compare("ddt_bias", to_np(dbias), rdb, shape.dtype_io)
    if two:
        compare("dlambda_logit", to_np(dlg), rdl, shape.dtype_io)


def test_composed_scan_from_raw_dt():
    """z -> dt (GPU pre-activation) -> scan forward, against the oracle scan of
    the oracle's dt."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=1, nheads=2, ngroups=2, seqlen=130)
    inp = S.make_inputs(shape, seed=21, with_dy=False)
    z, bias, logit = _raw(shape, 22)
    desc = abi.make_desc(shape)
    dev = scan.to_device(shape, inp)
    abi.ssm_preact_fwd(desc, _dev(z, shape), torch.from_numpy(bias).cuda(), _dev(logit, shape),
                       dev.dt, dev.lam)
    y, hT, _ = scan.scan_forward(shape, dev)
    torch.cuda.synchronize()
    rdt, rlam = oracle.preact_fwd(z, bias, logit)
    ref = oracle.scan_fwd(shape, dict(inp, dt=rdt, lam=rlam))
    compare("y", to_np(y), ref["y"], shape.dtype_io)
    compare("hT", to_np(hT), ref["hT"], shape.dtype_io)
