"""Sequence sharding on the GPU: a sequence cut into segments, each scanned by
the library with the boundary values of the others (the sharded algorithm,
its exchanges done by stacking on one device; no kernel waits on another),
gives the whole-sequence scan of the oracle: y, the final state and last
write, every token gradient, and the per-head parameter gradients summed
over segments."""
import numpy as np
import pytest

import oracle
from selective_diagonal_state_b200 import abi, cp, scan
from selective_diagonal_state_b200 import synthetic as S
from tests.parity_util import compare, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from selective_diagonal_state_b200 import build
    build.build()
    abi.load_library()


CASES = [
    # per-coordinate tensor-core chain: segments of 100 tokens (two chunks, ragged)
    ("hybridmamba", dict(batch=2, nheads=4, ngroups=4, seqlen=300), 3),
    # the same with the ZOH write, segments of unequal length
    ("hybridmamba", dict(batch=2, nheads=4, ngroups=4, seqlen=257, two_endpoint=0,
                         discretization=S.DISC_ZOH), 2),
    # recurrent kernels, fp32
    ("tiny_hybrid_fp32", dict(seqlen=90), 2),
    # scalar-decay chain: grouped heads, and rank 4 MIMO
    ("mamba2_siso", dict(batch=2, seqlen=400), 4),
    ("ssd_mimo_r4", dict(batch=1, nheads=2, ngroups=2, seqlen=200), 2),
    # channel scan
    ("mamba1_siso", dict(batch=2, nheads=64, seqlen=150), 3),
    # eight segments of 65 tokens (a full chunk and a one-token chunk each)
    ("hybridmamba", dict(batch=1, nheads=2, ngroups=2, seqlen=520), 8),
    # segments of one and two tokens, on the tensor-core chain and the recurrent kernels
    ("hybridmamba", dict(batch=1, nheads=2, ngroups=2, seqlen=10), 8),
    ("tiny_hybrid_fp32", dict(seqlen=9), 8),
    # many channels: the head-tiled segment transition
    ("mamba1_siso", dict(batch=1, nheads=320, seqlen=64), 2),
]


@pytest.mark.parametrize("name,kw,nseg", CASES)
def test_sharded_scan_matches_whole_sequence(name, kw, nseg):
    shape = S.WORKLOADS[name].replace(**kw)
    inp = S.make_inputs(shape, seed=31, with_state=True)
    segs, bounds = [], []
    for k in range(nseg):
        a, b = cp.segment_bounds(shape.seqlen, nseg, k)
        seg = cp.SegmentScan(shape.replace(seqlen=b - a))
        seg.load(inp, a, b)
        segs.append(seg)
        bounds.append((a, b))
    h0 = torch.from_numpy(inp["h0"]).cuda()
    w0 = torch.from_numpy(inp["w0"]).cuda()
    fwd, grads = cp.run_sharded(segs, h0=h0, w0=w0)
    torch.cuda.synchronize()
    abi.ssm_scan_poll_device_error()
    ref = oracle.scan_fwd(shape, inp)
    gr = oracle.scan_bwd(shape, inp, inp["dy"])
    dt = shape.dtype_io
    cat = lambda ts: np.concatenate([to_np(t) for t in ts], axis=1)  # noqa: E731
    lens = [b - a for a, b in bounds]
    compare("y", cat([f[0] for f in fwd]), ref["y"], dt)
    compare("hT", to_np(fwd[-1][1]), ref["hT"], dt)
    compare("last_write", to_np(fwd[-1][2]), ref["wT"], dt)
    compare("dx", cat([g.dx[:, :n] for g, n in zip(grads, lens)]), gr["dx"], dt)
    compare("ddt", cat([g.ddt[:, :n] for g, n in zip(grads, lens)]), gr["ddt"], dt)
    compare("dB", cat([g.dBm[:, :n] for g, n in zip(grads, lens)]), gr["dBm"], dt)
    compare("dC", cat([g.dCm[:, :n] for g, n in zip(grads, lens)]), gr["dCm"], dt)
    if shape.two_endpoint:
        compare("dlambda", cat([g.dlam[:, :n] for g, n in zip(grads, lens)]), gr["dlam"], dt)
    compare("dA_log", sum(to_np(g.dA_log) for g in grads), gr["dA_log"], dt)
    if shape.n_pairs:
        compare("dtheta", sum(to_np(g.dtheta) for g in grads), gr["dtheta"], dt)
    if shape.rank_in == shape.rank_out:
        compare("dD", sum(to_np(g.dD) for g in grads), gr["dD"], dt)
    compare("dh0", to_np(grads[0].dh0), gr["dh0"], dt)
    compare("dprev_write", to_np(grads[0].dw0), gr["dw0"], dt)


def test_one_segment_is_the_plain_scan():
    """nseg = 1: no boundary values enter; the result is the library's scan."""
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, nheads=4, ngroups=4, seqlen=130)
    inp = S.make_inputs(shape, seed=32, with_state=True)
    seg = cp.SegmentScan(shape)
    seg.load(inp, 0, shape.seqlen)
    fwd, grads = cp.run_sharded([seg], h0=torch.from_numpy(inp["h0"]).cuda(),
                                w0=torch.from_numpy(inp["w0"]).cuda())
    torch.cuda.synchronize()
    ref = oracle.scan_fwd(shape, inp)
    compare("y", to_np(fwd[0][0]), ref["y"], shape.dtype_io)
    gr = oracle.scan_bwd(shape, inp, inp["dy"])
    compare("dx", to_np(grads[0].dx[:, :shape.seqlen]), gr["dx"], shape.dtype_io)


@pytest.mark.parametrize("kw", [dict(), dict(angle_mode=S.ANGLE_PER_TOKEN), dict(n_static=16),
                                dict(two_endpoint=0),
                                # many heads: the head-tiled kernel, a partial last tile
                                dict(nheads=300, ngroups=300)])
def test_segment_transition(kw):
    """phi of a segment is the product of its tokens' transitions: e^{a sum dt} on a
    real row (e^{a L} on a static one), times a rotation by theta sum dt (or by the
    sum of the per-token angles) on a pair; beta_0 the first token's (1 - lam) dt."""
    kw = dict(dict(nheads=3, ngroups=3), **kw)
    shape = S.WORKLOADS["hybridmamba"].replace(batch=2, seqlen=77, **kw)
    H = shape.nheads
    inp = S.make_inputs(shape, seed=51)
    dev = scan.to_device(shape, inp)
    nmode = shape.n_real + shape.n_pairs
    phi = torch.empty((2, H, nmode, 2), dtype=torch.float32, device="cuda")
    beta0 = torch.empty((2, H), dtype=torch.float32, device="cuda")
    abi.ssm_cp_segment_transition(abi.make_desc(shape), dev.dt, dev.A_log, dev.theta, dev.lam,
                                  phi, beta0)
    torch.cuda.synchronize()
    a = -np.exp(inp["A_log"].astype(np.float64))                     # [H, nmode]
    sdt = inp["dt"].astype(np.float64).sum(axis=1)                    # [B, H]
    mag = np.exp(a[None] * sdt[:, :, None])
    mag[:, :, :shape.n_static] = np.exp(a[None, :, :shape.n_static] * shape.seqlen)
    if shape.angle_mode == S.ANGLE_PER_TOKEN:
        ang = inp["theta"].astype(np.float64).sum(axis=1)             # [B, H, np]
    else:
        ang = inp["theta"].astype(np.float64)[None] * sdt[:, :, None]
    ref = np.zeros((2, H, nmode, 2))
    ref[:, :, :shape.n_real, 0] = mag[:, :, :shape.n_real]
    ref[:, :, shape.n_real:, 0] = mag[:, :, shape.n_real:] * np.cos(ang)
    ref[:, :, shape.n_real:, 1] = mag[:, :, shape.n_real:] * np.sin(ang)
    np.testing.assert_allclose(to_np(phi), ref, rtol=2e-4, atol=1e-6)
    b0 = ((1.0 - inp["lam"][:, 0]) * inp["dt"][:, 0]) if shape.two_endpoint else np.zeros((2, H))
    np.testing.assert_allclose(to_np(beta0), b0, rtol=1e-5, atol=1e-7)
