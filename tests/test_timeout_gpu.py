"""The timeout path of the chained tensor-core kernels, exercised without a
fault: with a carry-wait limit of zero polls every carry wait of a call gives up,
the call stops early and reports SSM_ERR_TIMEOUT from the next device-error
poll, and the next call with the normal limit is parity-green again.  Nothing
here faults, traps or hangs the GPU: each wait returns after at most its
limit, and the kernels drain their outstanding copies before they exit."""
import pytest

import oracle
from selective_diagonal_state_b200 import abi, scan
from selective_diagonal_state_b200 import synthetic as S
from tests.parity_util import compare, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


# one shape per chained tensor-core chain: per-coordinate (HybridMamba) and
# scalar-decay (SSD-MIMO), each several chunks long
CASES = {
    "per_coordinate": (S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=320, nheads=4,
                                                          ngroups=4), abi.ROUTE_CHUNKED),
    "scalar_decay": (S.WORKLOADS["ssd_mimo_r4"].replace(batch=2, seqlen=150, nheads=4,
                                                         ngroups=4), abi.ROUTE_SSD),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    from selective_diagonal_state_b200 import build
    build.build()
    abi.load_library()
    shape, route = CASES[request.param]
    inp = S.make_inputs(shape, seed=61, with_state=True)
    return shape, inp, route


def _timed_out(fn):
    old = abi.ssm_scan_set_wait_limit(0)
    try:
        fn()
        with pytest.raises(abi.SsmError) as ei:
            abi.ssm_scan_poll_device_error()
        assert ei.value.code == -5   # SSM_ERR_TIMEOUT
    finally:
        abi.ssm_scan_set_wait_limit(old)
    abi.ssm_scan_poll_device_error()   # the error word was cleared by the poll


def test_forward_wait_gives_up_then_recovers(case):
    shape, inp, route = case
    dev = scan.to_device(shape, inp)
    if route == abi.ROUTE_SSD:
        # the scalar-decay forward walks whole segments and waits on no other work
        # item: with no polls allowed it still completes, with no error
        old = abi.ssm_scan_set_wait_limit(0)
        try:
            y, hT, wT = scan.scan_forward(shape, dev)
            torch.cuda.synchronize()
            abi.ssm_scan_poll_device_error()
        finally:
            abi.ssm_scan_set_wait_limit(old)
    else:
        _timed_out(lambda: scan.scan_forward(shape, dev))
        y, hT, wT = scan.scan_forward(shape, dev)
    assert abi.ssm_scan_last_route() == route
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(y), ref["y"], shape.dtype_io)
    compare("hT", to_np(hT), ref["hT"], shape.dtype_io)


def test_backward_wait_gives_up_then_recovers(case):
    shape, inp, route = case
    dev = scan.to_device(shape, inp)
    wsf = scan.alloc_workspace(shape, abi.PASS_FWD)
    scan.scan_forward(shape, dev, workspace=wsf)
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    _timed_out(lambda: scan.scan_backward(shape, dev, saved=wsf))
    g = scan.scan_backward(shape, dev, saved=wsf)
    assert abi.ssm_scan_last_route() == route
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    gr = oracle.scan_bwd(shape, inp, inp["dy"])
    for name, a, b in (("dx", g.dx, gr["dx"]), ("ddt", g.ddt, gr["ddt"]),
                       ("dB", g.dBm, gr["dBm"]), ("dC", g.dCm, gr["dCm"]),
                       ("dA_log", g.dA_log, gr["dA_log"]), ("dh0", g.dh0, gr["dh0"])):
        compare(name, to_np(a), b, shape.dtype_io)
