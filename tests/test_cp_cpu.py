"""Host side of sequence sharding (no GPU): segment bounds, the shapes that are
refused, the all-gather of boundary values over world-size-2 gloo ranks, and
the segment composition itself on the fp64 oracle."""
import os

import pytest

from selective_diagonal_state_b200 import cp
from selective_diagonal_state_b200 import synthetic as S

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("L,n", [(300, 3), (257, 2), (7, 4), (64, 1)])
def test_segment_bounds_tile_the_sequence(L, n):
    b = [cp.segment_bounds(L, n, k) for k in range(n)]
    assert b[0][0] == 0 and b[-1][1] == L
    assert all(b[k][1] == b[k + 1][0] for k in range(n - 1))
    lens = [hi - lo for lo, hi in b]
    assert max(lens) - min(lens) <= 1


def test_segment_bounds_reject_bad_index():
    with pytest.raises(ValueError):
        cp.segment_bounds(10, 2, 2)


@pytest.mark.parametrize("kw", [dict(angle_mode=S.ANGLE_PER_TOKEN), dict(n_static=8)])
def test_unsupported_shapes_are_refused(kw):
    shape = S.WORKLOADS["hybridmamba"].replace(batch=1, seqlen=64, **kw)
    with pytest.raises(ValueError):
        cp.SegmentScan(shape, device="cpu")


def _gather_worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = torch.full((2, 3), float(rank + 1))
        g = cp.all_gather_stacked(t, world)
        q.put((rank, g.tolist()))
    finally:
        dist.destroy_process_group()


def test_all_gather_stacks_in_rank_order():
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        g = res[r]
        assert [row[0][0] for row in g] == [1.0, 2.0]   # segment k at index k


def _segment_inputs(inp, a, b, h0=None, w0=None):
    tok = ("x", "dt", "Bm", "Cm", "lam", "dy")
    sub = {k: (v[:, a:b] if k in tok and v is not None else v) for k, v in inp.items()}
    sub["h0"], sub["w0"] = h0, w0
    return sub


def _apply_phi(X, mag, ang, nr):
    """Phi applied to states [B][H][N][P]: real rows scaled by e^{a S}; a pair's
    (re, im) rows multiplied by e^{a S} e^{i angle}."""
    import numpy as np
    Y = X.copy()
    Y[:, :, :nr] *= mag[:, :, :nr, None]
    re, im = X[:, :, nr::2], X[:, :, nr + 1::2]
    m, c, s = mag[:, :, nr:, None], np.cos(ang)[..., None], np.sin(ang)[..., None]
    Y[:, :, nr::2] = m * (c * re - s * im)
    Y[:, :, nr + 1::2] = m * (s * re + c * im)
    return Y


@pytest.mark.parametrize("nseg,kw", [(2, {}), (3, {}), (5, {}),
                                     # exact zero-order hold (single endpoint: beta_0 = 0)
                                     (3, dict(two_endpoint=0, discretization=S.DISC_ZOH))])
def test_segment_composition_on_the_oracle(nseg, kw):
    """The composition the sharded scan rests on, on the fp64 oracle alone:
    segments scanned from a zero state and joined by
    K_in(k+1) = Phi_k (K_in(k) + beta_0(k) W_in(k)) + hT_loc(k), W_in(k+1) = last
    write of segment k (Phi_k: e^{a sum dt} and the rotation by theta sum dt;
    beta_0(k) = (1 - lambda) dt of the segment's first token) give the whole
    sequence's final state and last write, and each segment scanned again from
    (K_in(k), W_in(k)) gives the whole sequence's y on its tokens."""
    import numpy as np

    import oracle
    shape = S.WORKLOADS["tiny_hybrid_fp32"].replace(seqlen=41, **kw)
    inp = S.make_inputs(shape, seed=61, with_state=True)
    whole = oracle.scan_fwd(shape, inp)
    a_rate = -np.exp(inp["A_log"].astype(np.float64))                 # [H, nmode]
    theta = inp["theta"].astype(np.float64)                            # [H, n_pairs]
    K, W = inp["h0"].astype(np.float64), inp["w0"].astype(np.float64)
    for k in range(nseg):
        a, b = cp.segment_bounds(shape.seqlen, nseg, k)
        seg = shape.replace(seqlen=b - a)
        # the exact forward of the segment from what enters it
        y = oracle.scan_fwd(seg, _segment_inputs(inp, a, b, K, W))["y"]
        np.testing.assert_allclose(y, whole["y"][:, a:b], rtol=1e-10, atol=1e-12)
        loc = oracle.scan_fwd(seg, _segment_inputs(inp, a, b))
        S_dt = inp["dt"][:, a:b].astype(np.float64).sum(axis=1)        # [B, H]
        mag = np.exp(a_rate[None] * S_dt[:, :, None])                  # [B, H, nmode]
        ang = theta[None] * S_dt[:, :, None]                           # [B, H, n_pairs]
        beta0 = np.zeros(inp["dt"][:, a].shape)                        # [B, H]
        if shape.two_endpoint:
            lam0, dt0 = (inp[k][:, a].astype(np.float64) for k in ("lam", "dt"))
            beta0 = (1.0 - lam0) * dt0
        K = _apply_phi(K + beta0[:, :, None, None] * W, mag, ang, shape.n_real) + loc["hT"]
        W = loc["wT"]
    np.testing.assert_allclose(K, whole["hT"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(W, whole["wT"], rtol=1e-10, atol=1e-12)


def test_backward_composition_on_the_oracle():
    """The backward half on the fp64 oracle alone.  The adjoint entering the end of
    segment k is dK_end(k) = dh0_loc(k+1) + Phi_{k+1}^T dK_end(k+1), where
    dh0_loc(k+1) is that segment's dh0 with no end adjoint.  Fed through trailing
    rows (dt = x = B = 0, lambda = 1, C rows e_n, dy rows the end adjoint), with
    beta_0(k+1) dK_end(k) added as the adjoint of the segment's last write, each
    segment's backward gives the whole sequence's gradients on its tokens.  The
    parameter gradients are the segments' sums, and dh0 / dprev_write are those
    of the first segment."""
    import numpy as np

    import oracle
    shape = S.WORKLOADS["tiny_hybrid_fp32"].replace(seqlen=37)
    nseg, N, nr = 3, shape.nstate, shape.n_real
    inp = S.make_inputs(shape, seed=62, with_state=True)
    whole = oracle.scan_bwd(shape, inp, inp["dy"])
    a_rate = -np.exp(inp["A_log"].astype(np.float64))
    theta = inp["theta"].astype(np.float64)
    bounds = [cp.segment_bounds(shape.seqlen, nseg, k) for k in range(nseg)]
    f64 = lambda v: v.astype(np.float64)  # noqa: E731

    def phi_of(a, b):
        S_dt = f64(inp["dt"][:, a:b]).sum(axis=1)
        return np.exp(a_rate[None] * S_dt[:, :, None]), theta[None] * S_dt[:, :, None]

    def beta0_of(a):
        return (1.0 - f64(inp["lam"][:, a])) * f64(inp["dt"][:, a])

    # forward: the states entering every segment (the forward composition)
    K, W = f64(inp["h0"]), f64(inp["w0"])
    enter = []
    for k, (a, b) in enumerate(bounds):
        enter.append((K, W))
        loc = oracle.scan_fwd(shape.replace(seqlen=b - a), _segment_inputs(inp, a, b))
        mag, ang = phi_of(a, b)
        K = _apply_phi(K + beta0_of(a)[:, :, None, None] * W, mag, ang, nr) + loc["hT"]
        W = loc["wT"]
    # backward: local dh0, then the end adjoints from the last segment back
    dh0_loc = [oracle.scan_bwd(shape.replace(seqlen=b - a), _segment_inputs(inp, a, b, *enter[k]),
                               inp["dy"][:, a:b])["dh0"] for k, (a, b) in enumerate(bounds)]
    dK_end = [None] * nseg
    dK_end[-1] = np.zeros_like(dh0_loc[0])
    for k in range(nseg - 2, -1, -1):
        a1, b1 = bounds[k + 1]
        mag, ang = phi_of(a1, b1)
        dK_end[k] = dh0_loc[k + 1] + _apply_phi(dK_end[k + 1], mag, -ang, nr)   # Phi^T
    sums = {n: 0.0 for n in ("dA_log", "dtheta", "dD")}
    for k, (a, b) in enumerate(bounds):
        L = b - a
        ext = shape.replace(seqlen=L + N)
        sub = _segment_inputs(inp, a, b, *enter[k])
        pad = lambda v: np.concatenate([v, np.zeros((v.shape[0], N) + v.shape[2:], v.dtype)],  # noqa: E731
                                       axis=1)
        for name in ("x", "dt", "Bm", "Cm"):
            sub[name] = pad(sub[name])
        sub["lam"] = np.concatenate([sub["lam"], np.ones((shape.batch, N, shape.nheads),
                                                         sub["lam"].dtype)], axis=1)
        for n in range(N):
            sub["Cm"][:, L + n, :, 0, n] = 1.0
        dy = pad(f64(inp["dy"][:, a:b]))                                # fp64: the end adjoint rows
        dy[:, L:, :, 0, :] = np.transpose(dK_end[k], (0, 2, 1, 3))     # row n <- dK_end[:, :, n]
        g = oracle.scan_bwd(ext, sub, dy)
        # the last write's adjoint: dx += B^T dW, dB += sum over the group's heads of dW x^T
        dW = (beta0_of(bounds[k + 1][0])[:, :, None, None] * dK_end[k]) if k + 1 < nseg \
            else np.zeros_like(dK_end[k])
        hpg = shape.nheads // shape.ngroups
        for h in range(shape.nheads):
            gi = h // hpg
            for r in range(shape.rank_in):
                Bl = f64(inp["Bm"][:, b - 1, gi, r])                    # [B, N]
                xl = f64(inp["x"][:, b - 1, h, r])                      # [B, P]
                g["dx"][:, L - 1, h, r] += np.einsum("bn,bnp->bp", Bl, dW[:, h])
                g["dBm"][:, L - 1, gi, r] += np.einsum("bnp,bp->bn", dW[:, h], xl)
        for name in ("dx", "ddt", "dBm", "dCm", "dlam"):
            np.testing.assert_allclose(g[name][:, :L], whole[name][:, a:b], rtol=1e-9, atol=1e-11,
                                       err_msg=f"segment {k} {name}")
        for name in sums:
            sums[name] = sums[name] + g[name]
        if k == 0:
            np.testing.assert_allclose(g["dh0"], whole["dh0"], rtol=1e-9, atol=1e-11)
            np.testing.assert_allclose(g["dw0"], whole["dw0"], rtol=1e-9, atol=1e-11)
    for name, v in sums.items():
        np.testing.assert_allclose(v, whole[name], rtol=1e-9, atol=1e-11, err_msg=name)
