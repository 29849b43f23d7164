"""Parity at the full sizes of the workloads, in the launch configuration the
benchmark times: a training forward into its workspace, then the backward that
reads it.  The oracle recomputes sampled independent pieces of each problem
(sampled heads, head groups or batch rows, always over the whole sequence)
and every output of those pieces is compared element by element, including
the per-head parameter gradients.

* HybridMamba (8 x 8192, 32 heads, 64 real + 32 rotation pairs, two-endpoint):
  B and C are per head, so a head is an independent problem.
* Mamba-2 recovery (4 x 2048, 24 heads in 3 groups of 8): B and C are shared
  by the 8 heads of a group, so a whole group is the independent piece
  (its dB, dC sum the group's heads).
* Mamba-1 recovery (8 x 4096, 2048 channels, B and C shared by all channels):
  one batch row with every channel gives that row's y, dx, ddt, dB, dC, hT;
  the per-channel parameter gradients (sums over the batch) come from every
  batch row of sampled channels.
* SSD-MIMO rank 4 (4 x 16384, 16 heads, B and C per head): sampled heads.
* Variants at the HybridMamba / SSD-MIMO sizes: per-token rotation angles and
  the ZOH write on the per-coordinate tensor-core chain, one target row per
  token (O = 1, R = 4) on the scalar-decay chain; sampled heads.
"""
import pytest

import oracle
from selective_diagonal_state_b200 import abi, scan
from selective_diagonal_state_b200 import synthetic as S
from tests.parity_util import compare, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

PER_TOKEN = ("x", "dt", "lam", "Bm", "Cm", "dy")


def _train_step(name, seed, **variant):
    """Training forward (saving workspace) + backward on the full workload (with
    the descriptor changes `variant`); outputs as float64 numpy arrays and the
    route both calls took."""
    from selective_diagonal_state_b200 import build
    build.build()
    abi.load_library()
    shape = S.WORKLOADS[name].replace(**variant)
    inp = S.make_inputs(shape, seed=seed)
    dev = scan.to_device(shape, inp)
    wsf = scan.alloc_workspace(shape, abi.PASS_FWD)
    y, hT, wT = scan.scan_forward(shape, dev, workspace=wsf)
    route_f = abi.ssm_scan_last_route()
    g = scan.scan_backward(shape, dev, saved=wsf)
    route_b = abi.ssm_scan_last_route()
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    out = dict(y=to_np(y), hT=to_np(hT), wT=to_np(wT), dx=to_np(g.dx), ddt=to_np(g.ddt),
               dB=to_np(g.dBm), dC=to_np(g.dCm), dA_log=to_np(g.dA_log), dD=to_np(g.dD),
               dlam=to_np(g.dlam) if g.dlam is not None else None,
               dtheta=to_np(g.dtheta) if g.dtheta is not None else None)
    del dev, wsf, y, hT, wT, g
    torch.cuda.empty_cache()
    return shape, inp, out, (route_f, route_b)


def _sub_inputs(inp, heads, groups=None, batch=None):
    """Inputs of the sub-problem made of `heads` (a slice), the B/C groups
    `groups` (a slice; None keeps every group) and the batch rows `batch`."""
    bsl = batch if batch is not None else slice(None)
    si = {}
    for k in PER_TOKEN:
        a = inp[k][bsl]
        if k in ("Bm", "Cm"):
            si[k] = a if groups is None else a[:, :, groups]
        else:
            si[k] = a[:, :, heads]
    th = inp["theta"]
    th = th[bsl][:, :, heads] if th.ndim == 4 else th[heads]   # per-token angles [B,L,H,np]
    si.update(A_log=inp["A_log"][heads], theta=th, D=inp["D"][heads])
    return si


def _check(prefix, shape, out, ref, grad, heads, groups=None, batch=None, fields=None):
    bsl = batch if batch is not None else slice(None)
    dt = shape.dtype_io
    gsl = groups if groups is not None else slice(None)
    pairs = {
        "y": (out["y"][bsl][:, :, heads], ref["y"]),
        "hT": (out["hT"][bsl][:, heads], ref["hT"]),
        "last_write": (out["wT"][bsl][:, heads], ref["wT"]),
        "dx": (out["dx"][bsl][:, :, heads], grad["dx"]),
        "ddt": (out["ddt"][bsl][:, :, heads], grad["ddt"]),
        "dB": (out["dB"][bsl][:, :, gsl], grad["dBm"]),
        "dC": (out["dC"][bsl][:, :, gsl], grad["dCm"]),
        "dA_log": (out["dA_log"][heads], grad["dA_log"]),
    }
    if shape.rank_in == shape.rank_out:
        pairs["dD"] = (out["dD"][heads], grad["dD"])
    if shape.two_endpoint:
        pairs["dlambda"] = (out["dlam"][bsl][:, :, heads], grad["dlam"])
    if shape.n_pairs:
        dth = out["dtheta"]
        pairs["dtheta"] = (dth[bsl][:, :, heads] if dth.ndim == 4 else dth[heads], grad["dtheta"])
    for k, (a, b) in pairs.items():
        if fields is None or k in fields:
            compare(k, a, b, dt)


# ---- HybridMamba -------------------------------------------------------------
@pytest.fixture(scope="module")
def hybrid_run():
    return _train_step("hybridmamba", seed=4)


@pytest.mark.parametrize("h", (0, 13, 31))
def test_hybridmamba_sampled_head(hybrid_run, h):
    shape, inp, out, routes = hybrid_run
    assert routes == (abi.ROUTE_CHUNKED, abi.ROUTE_CHUNKED)
    hs = slice(h, h + 1)
    sub = shape.replace(nheads=1, ngroups=1)
    si = _sub_inputs(inp, hs, groups=hs)
    _check("hybrid", shape, out, oracle.scan_fwd(sub, si), oracle.scan_bwd(sub, si, si["dy"]),
           hs, groups=hs)


# ---- Mamba-2 recovery (grouped B/C) ----------------------------------------------
@pytest.fixture(scope="module")
def mamba2_run():
    return _train_step("mamba2_siso", seed=5)


@pytest.mark.parametrize("g", (0, 2))
def test_mamba2_sampled_group(mamba2_run, g):
    shape, inp, out, routes = mamba2_run
    assert routes == (abi.ROUTE_SSD, abi.ROUTE_SSD)
    hpg = shape.nheads // shape.ngroups
    hs, gs = slice(g * hpg, (g + 1) * hpg), slice(g, g + 1)
    sub = shape.replace(nheads=hpg, ngroups=1)
    si = _sub_inputs(inp, hs, groups=gs)
    _check("mamba2", shape, out, oracle.scan_fwd(sub, si), oracle.scan_bwd(sub, si, si["dy"]),
           hs, groups=gs)


# ---- Mamba-1 recovery (B/C shared by every channel) ---------------------------------
@pytest.fixture(scope="module")
def mamba1_run():
    return _train_step("mamba1_siso", seed=6)


def test_mamba1_sampled_batch_row(mamba1_run):
    shape, inp, out, routes = mamba1_run
    assert routes == (abi.ROUTE_CHANNEL, abi.ROUTE_CHANNEL)
    b = 5
    bs = slice(b, b + 1)
    hs = slice(None)
    sub = shape.replace(batch=1)
    si = _sub_inputs(inp, hs, batch=bs)
    _check("mamba1", shape, out, oracle.scan_fwd(sub, si), oracle.scan_bwd(sub, si, si["dy"]),
           hs, batch=bs, fields=("y", "hT", "last_write", "dx", "ddt", "dB", "dC"))


@pytest.mark.parametrize("h", (0, 1000, 2047))
def test_mamba1_sampled_channel_params(mamba1_run, h):
    shape, inp, out, _ = mamba1_run
    hs = slice(h, h + 1)
    sub = shape.replace(nheads=1)
    si = _sub_inputs(inp, hs)
    grad = oracle.scan_bwd(sub, si, si["dy"])
    compare("dA_log", out["dA_log"][hs], grad["dA_log"], shape.dtype_io)
    compare("dD", out["dD"][hs], grad["dD"], shape.dtype_io)
    compare("ddt", out["ddt"][:, :, hs], grad["ddt"], shape.dtype_io)
    compare("dx", out["dx"][:, :, hs], grad["dx"], shape.dtype_io)


# ---- SSD-MIMO rank 4 -----------------------------------------------------------
@pytest.fixture(scope="module")
def mimo_run():
    return _train_step("ssd_mimo_r4", seed=7)


@pytest.mark.parametrize("h", (3, 15))
def test_mimo_sampled_head(mimo_run, h):
    shape, inp, out, routes = mimo_run
    assert routes == (abi.ROUTE_SSD, abi.ROUTE_SSD)
    hs = slice(h, h + 1)
    sub = shape.replace(nheads=1, ngroups=1)
    si = _sub_inputs(inp, hs, groups=hs)
    _check("mimo", shape, out, oracle.scan_fwd(sub, si), oracle.scan_bwd(sub, si, si["dy"]),
           hs, groups=hs)


# ---- variants at full size ----------------------------------------------------------
@pytest.fixture(scope="module")
def per_token_run():
    return _train_step("hybridmamba", seed=8, angle_mode=S.ANGLE_PER_TOKEN)


@pytest.mark.parametrize("h", (5, 30))
def test_per_token_angles_sampled_head(per_token_run, h):
    shape, inp, out, routes = per_token_run
    assert routes == (abi.ROUTE_CHUNKED, abi.ROUTE_CHUNKED)
    hs = slice(h, h + 1)
    sub = shape.replace(nheads=1, ngroups=1)
    si = _sub_inputs(inp, hs, groups=hs)
    _check("per-token", shape, out, oracle.scan_fwd(sub, si), oracle.scan_bwd(sub, si, si["dy"]),
           hs, groups=hs)


@pytest.fixture(scope="module")
def zoh_run():
    return _train_step("hybridmamba", seed=9, two_endpoint=0, discretization=S.DISC_ZOH)


@pytest.mark.parametrize("h", (2, 27))
def test_zoh_write_sampled_head(zoh_run, h):
    shape, inp, out, routes = zoh_run
    assert routes == (abi.ROUTE_CHUNKED, abi.ROUTE_CHUNKED)
    hs = slice(h, h + 1)
    sub = shape.replace(nheads=1, ngroups=1)
    si = _sub_inputs(inp, hs, groups=hs)
    _check("zoh", shape, out, oracle.scan_fwd(sub, si), oracle.scan_bwd(sub, si, si["dy"]),
           hs, groups=hs)


@pytest.fixture(scope="module")
def mimo_o1_run():
    return _train_step("ssd_mimo_r4", seed=10, rank_out=1)


def test_mimo_one_target_row_sampled_head(mimo_o1_run):
    shape, inp, out, routes = mimo_o1_run
    assert routes == (abi.ROUTE_SSD, abi.ROUTE_SSD)
    hs = slice(9, 10)
    sub = shape.replace(nheads=1, ngroups=1)
    si = _sub_inputs(inp, hs, groups=hs)
    _check("mimo-o1", shape, out, oracle.scan_fwd(sub, si), oracle.scan_bwd(sub, si, si["dy"]),
           hs, groups=hs)
