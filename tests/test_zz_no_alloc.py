"""The allocation-free backward entry point.

Some callers cannot call cudaMalloc (a host framework that owns all device
memory through its own pool, or a latency-critical path where allocating is
not allowed).  ssm_scan_bwd_noalloc serves them: it takes no workspace and
uses a fixed scratch array inside the library.  This file checks, through the
C ABI, that two calls in a row give the same gradients as ssm_scan_bwd with a
caller-provided workspace, and that a problem too large for the built-in
scratch is refused before any launch.  It is collected last on purpose.
"""
import pytest

from selective_diagonal_state_b200 import abi, scan
from selective_diagonal_state_b200 import synthetic as S
from tests.parity_util import compare, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

FIELDS = ["dx", "ddt", "dA_log", "dtheta", "dBm", "dCm", "dD", "dlam", "dh0", "dw0"]


def _noalloc(shape, dev, desc):
    g = scan.alloc_bwd(shape)
    abi.ssm_scan_bwd_noalloc(desc, dev.x, dev.dt, dev.A_log, dev.theta, dev.Bm, dev.Cm, dev.D,
                             dev.lam, dev.h0, dev.w0, dev.dy, g.dx, g.ddt, g.dA_log, g.dtheta,
                             g.dBm, g.dCm, g.dD, g.dlam, g.dh0, g.dw0)
    return g


@pytest.mark.parametrize("name,kw", [
    ("hybridmamba", dict(batch=2, seqlen=77, nheads=4, ngroups=4)),
    ("ssd_mimo_r4", dict(batch=1, seqlen=45, nheads=2, ngroups=2)),
    ("tiny_hybrid_fp32", dict()),
])
def test_noalloc_backward_matches_workspace_backward(name, kw):
    from selective_diagonal_state_b200 import build
    build.build()
    shape = S.WORKLOADS[name].replace(**kw)
    desc = abi.make_desc(shape)
    assert 0 < abi.ssm_scan_workspace_size(desc, abi.PASS_BWD) <= abi.NOALLOC_SCRATCH_BYTES
    inp = S.make_inputs(shape, seed=21, with_state=True)
    dev = scan.to_device(shape, inp)
    ref = scan.scan_backward(shape, dev, desc=desc)
    torch.cuda.synchronize()
    for _ in range(2):  # the scratch keeps the previous call's contents
        got = _noalloc(shape, dev, desc)
        torch.cuda.synchronize()
        abi.ssm_scan_poll_device_error()
        for f in FIELDS:
            a, b = getattr(got, f), getattr(ref, f)
            if b is None:
                continue
            compare(f, to_np(a), to_np(b), shape.dtype_io)


def test_noalloc_rejects_oversized_problem():
    shape = S.WORKLOADS["hybridmamba"].replace(batch=1, seqlen=4096)
    desc = abi.make_desc(shape)
    assert abi.ssm_scan_workspace_size(desc, abi.PASS_BWD) > abi.NOALLOC_SCRATCH_BYTES
    fake = 1 << 40  # never dereferenced: the size check fails first
    with pytest.raises(abi.SsmError) as ei:
        abi.ssm_scan_bwd_noalloc(desc, *([fake] * 21))
    assert ei.value.code == -6
