"""Pins for the fp64 oracle: each test checks it against something other than itself.

Every reference value below comes from a formulation the oracle does not
use (explicit transition-matrix products, a complex-mode recurrence, the
Vandermonde kernel and an FFT convolution, closed forms, the retrieval-rank
bound, central finite differences), so a dropped term, a wrong sign or index
or a transposed operand inside the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
from selective_diagonal_state_b200 import synthetic as S

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def tiny(**kw):
    base = dict(batch=2, seqlen=11, nheads=2, headdim=3, ngroups=2, n_real=3, n_pairs=2,
                rank_in=1, rank_out=1, decay_mode=S.DECAY_PER_COORD, two_endpoint=1,
                dtype_io=S.DTYPE_F32)
    base.update(kw)
    return S.ScanShape(**base)


def inputs(shape, seed=0, state=True):
    inp = S.make_inputs(shape, seed, with_dy=True, with_state=state)
    # widen the step so decays and rotations are far from the identity
    inp["dt"] = (inp["dt"] * 20.0 + 0.05).astype(np.float32)
    return {k: v.astype(np.float64) for k, v in inp.items()}


# ---------------------------------------------------------------------------
# independent building blocks (explicit matrices / complex modes)
# ---------------------------------------------------------------------------
def decay_rate(shape, A_log, h, k):
    """a for decay slot k of head h."""
    return -math.exp(A_log[h, k if shape.decay_mode == S.DECAY_PER_COORD else 0])


def transition_matrix(shape, inp, b, t, h):
    """The N x N transition of step t as an explicit matrix."""
    N = shape.nstate
    T = np.zeros((N, N))
    dt = inp["dt"][b, t, h]
    for n in range(shape.n_real):
        T[n, n] = math.exp(dt * decay_rate(shape, inp["A_log"], h, n))
    for j in range(shape.n_pairs):
        r = shape.n_real + 2 * j
        e = math.exp(dt * decay_rate(shape, inp["A_log"], h, shape.n_real + j))
        ph = dt * inp["theta"][h, j]
        T[r:r + 2, r:r + 2] = e * np.array([[math.cos(ph), -math.sin(ph)],
                                            [math.sin(ph), math.cos(ph)]])
    return T


def weights(shape, inp, b, t, h):
    dt = inp["dt"][b, t, h]
    lam = inp["lam"][b, t, h] if shape.two_endpoint else 1.0
    return lam * dt, (1.0 - lam) * dt


def group_of(shape, h):
    return h // (shape.nheads // shape.ngroups)


def quadratic_form(shape, inp):
    """y_t = sum_{s<=t} c_{t,s} C_t Phi_{t,s} B_s u_s + C_t Phi_{t,-1} (h0 + beta_0 w0) + D u_t.

    Phi_{t,s} = T_t ... T_{s+1} built by explicit matrix products; the weight of
    source s is gamma_s (s = t) or gamma_s + beta_{s+1} (s < t): the masked
    state-mediated kernel of the linear-attention view.
    """
    Bt, L, H, P = shape.batch, shape.seqlen, shape.nheads, shape.headdim
    N, R, O = shape.nstate, shape.rank_in, shape.rank_out
    y = np.zeros((Bt, L, H, O, P))
    hT = np.zeros((Bt, H, N, P))
    for b in range(Bt):
        for h in range(H):
            g = group_of(shape, h)
            Ts = [transition_matrix(shape, inp, b, t, h) for t in range(L)]
            gb = [weights(shape, inp, b, t, h) for t in range(L)]

            def phi(t, s):
                M = np.eye(N)
                for k in range(s + 1, t + 1):
                    M = Ts[k] @ M
                return M

            init = inp["h0"][b, h] + gb[0][1] * inp["w0"][b, h]
            for t in range(L + 1):
                tt = min(t, L - 1)
                acc = phi(tt, -1) @ init
                for s in range(tt + 1):
                    w = gb[s][0] + (gb[s + 1][1] if s < tt else 0.0)
                    Bs = inp["Bm"][b, s, g].T          # N x R
                    acc = acc + w * phi(tt, s) @ Bs @ inp["x"][b, s, h]
                if t == L:
                    hT[b, h] = acc
                    break
                Ct = inp["Cm"][b, t, g]                 # O x N
                y[b, t, h] = Ct @ acc
                if O == R:
                    y[b, t, h] += inp["D"][h] * inp["x"][b, t, h]
    return y, hT


@pytest.mark.parametrize("kw", [
    dict(),
    dict(decay_mode=S.DECAY_PER_HEAD),
    dict(rank_in=2, rank_out=2, ngroups=1),
    dict(rank_in=3, rank_out=2, n_pairs=1),
    dict(two_endpoint=0, n_pairs=0, n_real=4),
    dict(nheads=4, ngroups=2, batch=1),
])
def test_recurrence_equals_quadratic_masked_form(kw):
    """Thm 24 view (sungsoo.github.io Part 03): the state-mediated kernel is masked
    unnormalised linear attention, initial state and feedthrough included."""
    sh = tiny(**kw)
    inp = inputs(sh, seed=1)
    out = oracle.scan_fwd(sh, inp)
    yq, hq = quadratic_form(sh, inp)
    np.testing.assert_allclose(out["y"], yq, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(out["hT"], hq, rtol=1e-11, atol=1e-11)


def complex_modes(shape, inp):
    """Complex-diagonal recurrence: one complex mode per real row (eigenvalue real) and
    per rotation pair (eigenvalue exp(dt (a + i theta))), y = sum Re(conj(c) z)."""
    Bt, L, H, P = shape.batch, shape.seqlen, shape.nheads, shape.headdim
    nr, npr, R, O = shape.n_real, shape.n_pairs, shape.rank_in, shape.rank_out
    y = np.zeros((Bt, L, H, O, P))
    for b in range(Bt):
        for h in range(H):
            g = group_of(shape, h)
            lam_mode = []
            for n in range(nr):
                lam_mode.append(complex(decay_rate(shape, inp["A_log"], h, n), 0.0))
            for j in range(npr):
                lam_mode.append(complex(decay_rate(shape, inp["A_log"], h, nr + j),
                                        inp["theta"][h, j]))
            lam_mode = np.array(lam_mode)

            def to_c(v):  # N-vector (rows) -> complex mode vector
                return np.concatenate([v[:nr] + 0j, v[nr::2][:npr] + 1j * v[nr + 1::2][:npr]])

            z = np.stack([to_c(inp["h0"][b, h][:, p]) for p in range(P)], axis=1)
            wp = np.stack([to_c(inp["w0"][b, h][:, p]) for p in range(P)], axis=1)
            for t in range(L):
                dt = inp["dt"][b, t, h]
                gam, bet = weights(shape, inp, b, t, h)
                eig = np.exp(dt * lam_mode)[:, None]
                bm = np.stack([to_c(inp["Bm"][b, t, g, r]) for r in range(R)], axis=1)
                w = bm @ inp["x"][b, t, h]
                z = eig * (z + bet * wp) + gam * w
                for o in range(O):
                    c = to_c(inp["Cm"][b, t, g, o])
                    y[b, t, h, o] = np.real(np.conj(c)[:, None] * z).sum(0)
                if O == R:
                    y[b, t, h] += inp["D"][h] * inp["x"][b, t, h]
                wp = w
    return y


@pytest.mark.parametrize("kw", [dict(), dict(n_real=0, n_pairs=3), dict(rank_in=2, rank_out=2)])
def test_real_2x2_blocks_equal_complex_diagonal(kw):
    """Thm 8 (sungsoo.github.io Part 03): over the reals a complex eigenvalue pair is a
    2x2 decay-rotation block; the block recurrence must equal the complex one."""
    sh = tiny(**kw)
    inp = inputs(sh, seed=2)
    out = oracle.scan_fwd(sh, inp)
    np.testing.assert_allclose(out["y"], complex_modes(sh, inp), rtol=1e-11, atol=1e-11)


def test_rotary_identity():
    """exp(i w (S_t - S_s)) = exp(i w S_t) exp(-i w S_s) for the pair phases."""
    rng = np.random.default_rng(0)
    w = rng.uniform(0, math.pi, 5)
    St, Ss = rng.uniform(0, 10, 2)
    np.testing.assert_allclose(np.exp(1j * w * (St - Ss)),
                               np.exp(1j * w * St) * np.exp(-1j * w * Ss), rtol=1e-13)


def test_lti_equals_vandermonde_convolution():
    """With dt, lam, B, C fixed in time the scan is a convolution with
    K_0 = gamma C.B and K_k = (gamma + beta) Re(conj(c) a^k b) (Vandermonde in the
    eigenvalues a): robocikowo.com glossary item 3 and the S4D kernel."""
    sh = tiny(batch=1, seqlen=40, nheads=2, headdim=2, n_real=4, n_pairs=3)
    inp = inputs(sh, seed=3, state=False)
    L = sh.seqlen
    for key in ("dt", "lam"):
        inp[key] = np.broadcast_to(inp[key][:, :1], inp[key].shape).copy()
    for key in ("Bm", "Cm"):
        inp[key] = np.broadcast_to(inp[key][:, :1], inp[key].shape).copy()
    y = oracle.scan_fwd(sh, inp)["y"]
    nr, npr = sh.n_real, sh.n_pairs
    for h in range(sh.nheads):
        g = group_of(sh, h)
        dt = inp["dt"][0, 0, h]
        gam, bet = weights(sh, inp, 0, 0, h)
        eig = np.array([decay_rate(sh, inp["A_log"], h, n) + 0j for n in range(nr)] +
                       [complex(decay_rate(sh, inp["A_log"], h, nr + j), inp["theta"][h, j])
                        for j in range(npr)])
        a = np.exp(dt * eig)
        bv, cv = inp["Bm"][0, 0, g, 0], inp["Cm"][0, 0, g, 0]
        bc = np.concatenate([bv[:nr] + 0j, bv[nr::2] + 1j * bv[nr + 1::2]])
        cc = np.concatenate([cv[:nr] + 0j, cv[nr::2] + 1j * cv[nr + 1::2]])
        V = a[:, None] ** np.arange(L)[None, :]            # Vandermonde
        K = np.real((np.conj(cc) * bc) @ V) * (gam + bet)
        K[0] = gam * np.real(np.conj(cc) @ bc)
        for p in range(sh.headdim):
            u = inp["x"][0, :, h, 0, p]
            n = 2 * L
            conv = np.fft.irfft(np.fft.rfft(K, n) * np.fft.rfft(u, n), n)[:L]
            np.testing.assert_allclose(y[0, :, h, 0, p], conv + inp["D"][h] * u,
                                       rtol=1e-9, atol=1e-10)


def test_no_decay_is_unnormalised_linear_attention():
    """a -> 0, theta = 0, lam = 1: y = (tril(C B^T) diag(dt)) X + D X (kongchang.com
    "Connection to Linear Attention")."""
    sh = tiny(two_endpoint=0, nheads=2, ngroups=1, seqlen=9)
    inp = inputs(sh, seed=4, state=False)
    inp["A_log"][:] = -80.0
    inp["theta"][:] = 0.0
    y = oracle.scan_fwd(sh, inp)["y"]
    for b in range(sh.batch):
        for h in range(sh.nheads):
            C = inp["Cm"][b, :, 0, 0]
            B = inp["Bm"][b, :, 0, 0]
            X = inp["x"][b, :, h, 0]
            att = np.tril(C @ B.T) * inp["dt"][b, :, h][None, :]
            np.testing.assert_allclose(y[b, :, h, 0], att @ X + inp["D"][h] * X,
                                       rtol=1e-12, atol=1e-12)


def test_scalar_decay_is_segsum_masked_attention():
    """Mamba-2 special case: one decay per head gives the segment-sum mask
    L[t,s] = exp(a (S_t - S_s)), y = (L * C B^T) diag(dt) X + D X."""
    sh = tiny(decay_mode=S.DECAY_PER_HEAD, two_endpoint=0, n_pairs=0, n_real=5,
              nheads=4, ngroups=2, seqlen=13, headdim=4)
    inp = inputs(sh, seed=5, state=False)
    y = oracle.scan_fwd(sh, inp)["y"]
    for b in range(sh.batch):
        for h in range(sh.nheads):
            g = group_of(sh, h)
            a = decay_rate(sh, inp["A_log"], h, 0)
            cs = np.cumsum(inp["dt"][b, :, h])
            Lm = np.tril(np.exp(a * (cs[:, None] - cs[None, :])))
            C, B, X = inp["Cm"][b, :, g, 0], inp["Bm"][b, :, g, 0], inp["x"][b, :, h, 0]
            ref = (Lm * (C @ B.T)) @ (inp["dt"][b, :, h][:, None] * X) + inp["D"][h] * X
            np.testing.assert_allclose(y[b, :, h, 0], ref, rtol=1e-11, atol=1e-12)


def test_mamba1_per_coordinate_closed_form():
    """Mamba-1 special case (P = 1 channels, per-coordinate decay, shared B/C):
    y_t = sum_s sum_n C_tn exp(a_n (S_t - S_s)) dt_s B_sn x_s + D x_t."""
    sh = tiny(nheads=3, ngroups=1, headdim=1, n_real=4, n_pairs=0, two_endpoint=0,
              seqlen=10)
    inp = inputs(sh, seed=6, state=False)
    y = oracle.scan_fwd(sh, inp)["y"]
    for b in range(sh.batch):
        for h in range(sh.nheads):
            cs = np.cumsum(inp["dt"][b, :, h])
            x = inp["x"][b, :, h, 0, 0]
            for t in range(sh.seqlen):
                acc = 0.0
                for s in range(t + 1):
                    for n in range(sh.n_real):
                        a = decay_rate(sh, inp["A_log"], h, n)
                        acc += (inp["Cm"][b, t, 0, 0, n] * math.exp(a * (cs[t] - cs[s])) *
                                inp["dt"][b, s, h] * inp["Bm"][b, s, 0, 0, n] * x[s])
                assert abs(y[b, t, h, 0, 0] - (acc + inp["D"][h] * x[t])) < 1e-11


def test_single_step_closed_form():
    """L = 1 from a zero state: y_0 = gamma_0 C_0 B_0 u_0 + D u_0."""
    sh = tiny(seqlen=1, rank_in=2, rank_out=2)
    inp = inputs(sh, seed=7, state=False)
    y = oracle.scan_fwd(sh, inp)["y"]
    for b in range(sh.batch):
        for h in range(sh.nheads):
            g = group_of(sh, h)
            gam = inp["lam"][b, 0, h] * inp["dt"][b, 0, h]
            ref = gam * inp["Cm"][b, 0, g] @ inp["Bm"][b, 0, g].T @ inp["x"][b, 0, h]
            ref += inp["D"][h] * inp["x"][b, 0, h]
            np.testing.assert_allclose(y[b, 0, h], ref, rtol=1e-12, atol=1e-13)


def test_carry_continuation():
    """Scan(0:L) == Scan(L1:L) started from (hT, last write) of Scan(0:L1)."""
    sh = tiny(seqlen=14)
    inp = inputs(sh, seed=8)
    full = oracle.scan_fwd(sh, inp)
    L1 = 6
    first = {k: (v[:, :L1] if k in ("x", "dt", "lam", "Bm", "Cm") else v) for k, v in inp.items()}
    a = oracle.scan_fwd(sh.replace(seqlen=L1), first)
    second = {k: (v[:, L1:] if k in ("x", "dt", "lam", "Bm", "Cm") else v) for k, v in inp.items()}
    second["h0"], second["w0"] = a["hT"], a["wT"]
    c = oracle.scan_fwd(sh.replace(seqlen=sh.seqlen - L1), second)
    np.testing.assert_allclose(np.concatenate([a["y"], c["y"]], 1), full["y"], rtol=1e-12,
                               atol=1e-12)
    np.testing.assert_allclose(c["hT"], full["hT"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("R,O", [(3, 3), (3, 2), (1, 1)])
def test_local_retrieval_rank(R, O):
    """Thm 21 (sungsoo.github.io Part 01 and Part 08 item 2): rank dy_t/du_s <= min(O, rank B_s),
    with equality for generic readouts; a rank-k B_s caps it at k."""
    sh = tiny(batch=1, nheads=1, ngroups=1, headdim=1, rank_in=R, rank_out=O, seqlen=6,
              n_real=4, n_pairs=2)
    inp = inputs(sh, seed=9, state=False)
    low = 2  # time step whose B gets rank 1
    v = np.random.default_rng(0).standard_normal((sh.nstate, 1))
    w = np.random.default_rng(1).standard_normal((1, R))
    inp["Bm"][0, low, 0] = (v @ w).T
    L = sh.seqlen

    def jac(t, s):
        J = np.zeros((O, R))
        for r in range(R):
            probe = dict(inp)
            probe["x"] = np.zeros_like(inp["x"])
            probe["x"][0, s, 0, r, 0] = 1.0
            probe["D"] = np.zeros_like(inp["D"])
            J[:, r] = oracle.scan_fwd(sh, probe)["y"][0, t, 0, :, 0]
        return J

    for s in range(L - 1):
        J = jac(L - 1, s)
        rank = np.linalg.matrix_rank(J, tol=1e-10)
        expect = min(O, R, 1 if s == low else R)
        assert rank == expect, (s, rank, expect)


# ---------------------------------------------------------------------------
# backward: central finite differences of <dy, y>
# ---------------------------------------------------------------------------
def _loss(shape, inp):
    out = oracle.scan_fwd(shape, inp)
    return float((out["y"] * inp["dy"]).sum())


GRAD_KEYS = [("x", "dx"), ("dt", "ddt"), ("A_log", "dA_log"), ("theta", "dtheta"),
             ("Bm", "dBm"), ("Cm", "dCm"), ("D", "dD"), ("lam", "dlam"), ("h0", "dh0"),
             ("w0", "dw0")]


@pytest.mark.parametrize("kw", [
    dict(rank_in=2, rank_out=2, ngroups=1),
    dict(rank_in=2, rank_out=2, ngroups=2),
    dict(decay_mode=S.DECAY_PER_HEAD),
    dict(rank_in=2, rank_out=1, two_endpoint=0),
    dict(nheads=4, ngroups=2, headdim=1, seqlen=8),
])
def test_gradients_match_central_differences(kw):
    base = dict(batch=1, seqlen=12, nheads=2, headdim=2, n_real=4, n_pairs=2)
    base.update(kw)
    sh = tiny(**base)
    inp = inputs(sh, seed=10)
    g = oracle.scan_bwd(sh, inp, inp["dy"])
    eps = 1e-6
    rng = np.random.default_rng(0)
    for key, gkey in GRAD_KEYS:
        if key == "lam" and not sh.two_endpoint:
            continue
        arr = inp[key]
        flat = arr.reshape(-1)
        idx = rng.choice(flat.size, size=min(flat.size, 24), replace=False)
        for i in idx:
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(sh, inp)
            flat[i] = old - eps
            lm = _loss(sh, inp)
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            an = g[gkey].reshape(-1)[i]
            scale = max(1.0, abs(fd))
            assert abs(fd - an) <= 1e-6 * scale, (key, i, fd, an)


# ---------------------------------------------------------------------------
# per-token rotation angles (the data-dependent angles of Mamba-3's complex
# state, sungsoo.github.io Part 05)
# ---------------------------------------------------------------------------
def test_per_token_angles_reduce_to_static_angles():
    """theta_t = dt_t theta_j gives the static-angle scan exactly, and the
    gradients split by the chain rule: ddt_static = ddt + sum_j theta_j dtheta_t,
    dtheta_static = sum_{b,t} dt_t dtheta_t; every other gradient is unchanged."""
    sh = tiny(n_real=3, n_pairs=2)
    inp = inputs(sh, seed=12)
    pt = sh.replace(angle_mode=1)
    ip = dict(inp)
    ip["theta"] = inp["dt"][..., None] * inp["theta"][None, None]
    ys, yp = oracle.scan_fwd(sh, inp), oracle.scan_fwd(pt, ip)
    np.testing.assert_allclose(yp["y"], ys["y"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(yp["hT"], ys["hT"], rtol=1e-12, atol=1e-12)
    gs, gp = oracle.scan_bwd(sh, inp, inp["dy"]), oracle.scan_bwd(pt, ip, ip["dy"])
    assert gp["dtheta"].shape == (sh.batch, sh.seqlen, sh.nheads, sh.n_pairs)
    np.testing.assert_allclose(gp["ddt"] + (gp["dtheta"] * inp["theta"][None, None]).sum(-1),
                               gs["ddt"], rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose((gp["dtheta"] * inp["dt"][..., None]).sum((0, 1)), gs["dtheta"],
                               rtol=1e-10, atol=1e-10)
    for k in ("dx", "dBm", "dCm", "dA_log", "dD", "dlam", "dh0", "dw0"):
        np.testing.assert_allclose(gp[k], gs[k], rtol=1e-10, atol=1e-10, err_msg=k)


def test_per_token_angles_equal_complex_modes():
    """The 2x2 blocks with per-token angles against a complex-mode recurrence
    whose eigenvalue of step t is exp(dt_t a + i theta_t)."""
    sh = tiny(n_real=2, n_pairs=3, angle_mode=1)
    inp = inputs(sh, seed=13)
    out = oracle.scan_fwd(sh, inp)
    Bt, L, H, P = sh.batch, sh.seqlen, sh.nheads, sh.headdim
    nr, npr = sh.n_real, sh.n_pairs
    y = np.zeros_like(out["y"])
    for b in range(Bt):
        for h in range(H):
            g = group_of(sh, h)
            a = np.array([decay_rate(sh, inp["A_log"], h, m) for m in range(nr + npr)])

            def to_c(v):
                return np.concatenate([v[:nr] + 0j, v[nr::2][:npr] + 1j * v[nr + 1::2][:npr]])

            z = np.stack([to_c(inp["h0"][b, h][:, p]) for p in range(P)], axis=1)
            wp = np.stack([to_c(inp["w0"][b, h][:, p]) for p in range(P)], axis=1)
            for t in range(L):
                dt = inp["dt"][b, t, h]
                gam, bet = weights(sh, inp, b, t, h)
                ph = np.concatenate([np.zeros(nr), inp["theta"][b, t, h]])
                eig = np.exp(dt * a + 1j * ph)[:, None]
                w = to_c(inp["Bm"][b, t, g, 0])[:, None] * inp["x"][b, t, h, 0][None, :]
                z = eig * (z + bet * wp) + gam * w
                c = to_c(inp["Cm"][b, t, g, 0])
                y[b, t, h, 0] = np.real(np.conj(c)[:, None] * z).sum(0) + inp["D"][h] * inp["x"][b, t, h, 0]
                wp = w
    np.testing.assert_allclose(out["y"], y, rtol=1e-11, atol=1e-11)


def test_per_token_angle_gradients_match_central_differences():
    sh = tiny(batch=1, seqlen=12, nheads=2, headdim=2, n_real=2, n_pairs=2, angle_mode=1)
    inp = inputs(sh, seed=14)
    g = oracle.scan_bwd(sh, inp, inp["dy"])
    eps = 1e-6
    rng = np.random.default_rng(1)
    for key, gkey in (("theta", "dtheta"), ("dt", "ddt"), ("A_log", "dA_log"), ("lam", "dlam")):
        flat = inp[key].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 24), replace=False):
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(sh, inp)
            flat[i] = old - eps
            lm = _loss(sh, inp)
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            an = g[gkey].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (key, i, fd, an)


# ---------------------------------------------------------------------------
# real static rows (HybridMamba's row types: real static, real dynamic and
# complex dynamic, sungsoo.github.io Part 08 item 3)
# ---------------------------------------------------------------------------
def test_static_rows_lti_vandermonde():
    """dt, lam, B, C fixed in time: a convolution whose Vandermonde eigenvalues
    are e^{a_n} on static rows (whatever dt) and e^{dt lam_n} on the others."""
    sh = tiny(batch=1, seqlen=40, nheads=2, headdim=2, n_real=5, n_pairs=2, n_static=3)
    inp = inputs(sh, seed=21, state=False)
    L = sh.seqlen
    for key in ("dt", "lam", "Bm", "Cm"):
        inp[key] = np.broadcast_to(inp[key][:, :1], inp[key].shape).copy()
    inp["dt"][:] = 0.3       # a step away from 1: static and dynamic rows differ
    y = oracle.scan_fwd(sh, inp)["y"]
    nr, npr = sh.n_real, sh.n_pairs
    for h in range(sh.nheads):
        g = group_of(sh, h)
        dt = inp["dt"][0, 0, h]
        gam, bet = weights(sh, inp, 0, 0, h)
        lam = np.array([decay_rate(sh, inp["A_log"], h, n) + 0j for n in range(nr)] +
                       [complex(decay_rate(sh, inp["A_log"], h, nr + j), inp["theta"][h, j])
                        for j in range(npr)])
        scale = np.array([1.0 if n < sh.n_static else dt for n in range(nr + npr)])
        a = np.exp(scale * lam)
        bv, cv = inp["Bm"][0, 0, g, 0], inp["Cm"][0, 0, g, 0]
        bc = np.concatenate([bv[:nr] + 0j, bv[nr::2] + 1j * bv[nr + 1::2]])
        cc = np.concatenate([cv[:nr] + 0j, cv[nr::2] + 1j * cv[nr + 1::2]])
        V = a[:, None] ** np.arange(L)[None, :]
        K = np.real((np.conj(cc) * bc) @ V) * (gam + bet)
        K[0] = gam * np.real(np.conj(cc) @ bc)
        for p in range(sh.headdim):
            u = inp["x"][0, :, h, 0, p]
            n = 2 * L
            conv = np.fft.irfft(np.fft.rfft(K, n) * np.fft.rfft(u, n), n)[:L]
            np.testing.assert_allclose(y[0, :, h, 0, p], conv + inp["D"][h] * u,
                                       rtol=1e-9, atol=1e-10)


def test_static_rows_equal_dynamic_rows_at_unit_step():
    """With dt_t = 1 everywhere a static row and a dynamic row are the same row:
    equal outputs and decay gradients; ddt loses exactly the static rows' a g_rho."""
    sh = tiny(n_real=6, n_pairs=2, two_endpoint=1)
    inp = inputs(sh, seed=22)
    inp["dt"][:] = 1.0
    st = sh.replace(n_static=4)
    y0, y1 = oracle.scan_fwd(sh, inp), oracle.scan_fwd(st, inp)
    np.testing.assert_allclose(y1["y"], y0["y"], rtol=1e-12, atol=1e-12)
    g0, g1 = oracle.scan_bwd(sh, inp, inp["dy"]), oracle.scan_bwd(st, inp, inp["dy"])
    for k in ("dx", "dBm", "dCm", "dA_log", "dtheta", "dD", "dlam", "dh0", "dw0"):
        np.testing.assert_allclose(g1[k], g0[k], rtol=1e-10, atol=1e-10, err_msg=k)
    assert np.abs(g1["ddt"] - g0["ddt"]).max() > 1e-3


@pytest.mark.parametrize("decay_mode", [S.DECAY_PER_COORD, S.DECAY_PER_HEAD])
def test_static_row_gradients_match_central_differences(decay_mode):
    sh = tiny(batch=1, seqlen=12, nheads=2, headdim=2, n_real=4, n_pairs=2, n_static=2,
              decay_mode=decay_mode)
    inp = inputs(sh, seed=23)
    g = oracle.scan_bwd(sh, inp, inp["dy"])
    eps = 1e-6
    rng = np.random.default_rng(2)
    for key, gkey in (("A_log", "dA_log"), ("dt", "ddt"), ("Bm", "dBm"), ("x", "dx")):
        flat = inp[key].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 16), replace=False):
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(sh, inp)
            flat[i] = old - eps
            lm = _loss(sh, inp)
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            an = g[gkey].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (key, i, fd, an)


# ---------------------------------------------------------------------------
# exact zero-order-hold discretisation (robocikowo.com glossary item 2)
# ---------------------------------------------------------------------------
def _continuous_A(shape, inp, b, t, h):
    """Real N x N generator of the continuous system of head h at step t:
    a_n on real rows, [[a, -w], [w, a]] on pair j (w = theta_j, or the
    per-token angle divided by the step)."""
    nr, npr, N = shape.n_real, shape.n_pairs, shape.nstate
    A = np.zeros((N, N))
    dt = inp["dt"][b, t, h]
    for n in range(nr):
        A[n, n] = decay_rate(shape, inp["A_log"], h, n)
    for j in range(npr):
        a = decay_rate(shape, inp["A_log"], h, nr + j)
        w = (inp["theta"][b, t, h, j] / dt if shape.angle_mode == S.ANGLE_PER_TOKEN
             else inp["theta"][h, j])
        r = nr + 2 * j
        A[r:r + 2, r:r + 2] = [[a, -w], [w, a]]
    return A


@pytest.mark.parametrize("kw", [dict(), dict(angle_mode=S.ANGLE_PER_TOKEN),
                                dict(decay_mode=S.DECAY_PER_HEAD, n_pairs=0)])
def test_zoh_equals_matrix_exponential(kw):
    """Zero-order hold is exact for an input held over the step: the step's
    transition and write are the blocks of expm([[A, I], [0, 0]] dt) (Van
    Loan), computed here by scipy's matrix exponential on the real 2x2 form."""
    from scipy.linalg import expm
    sh = tiny(two_endpoint=0, discretization=S.DISC_ZOH, **kw)
    inp = inputs(sh, seed=31)
    out = oracle.scan_fwd(sh, inp)
    N, P = sh.nstate, sh.headdim
    y = np.zeros_like(out["y"])
    for b in range(sh.batch):
        for h in range(sh.nheads):
            g = group_of(sh, h)
            H = inp["h0"][b, h].copy()
            for t in range(sh.seqlen):
                M = np.zeros((2 * N, 2 * N))
                M[:N, :N] = _continuous_A(sh, inp, b, t, h)
                M[:N, N:] = np.eye(N)
                E = expm(M * inp["dt"][b, t, h])
                W = inp["Bm"][b, t, g, 0][:, None] * inp["x"][b, t, h, 0][None, :]
                H = E[:N, :N] @ H + E[:N, N:] @ W
                y[b, t, h, 0] = inp["Cm"][b, t, g, 0] @ H + inp["D"][h] * inp["x"][b, t, h, 0]
    np.testing.assert_allclose(out["y"], y, rtol=1e-10, atol=1e-10)


def test_zoh_tends_to_euler_for_slow_modes():
    """|dt lam| -> 0: (e^{dt lam} - 1) / lam -> dt, the Euler write."""
    sh = tiny(two_endpoint=0)
    inp = inputs(sh, seed=32)
    inp["A_log"][:] = -30.0
    inp["theta"][:] = 1e-12
    a = oracle.scan_fwd(sh, inp)["y"]
    b = oracle.scan_fwd(sh.replace(discretization=S.DISC_ZOH), inp)["y"]
    np.testing.assert_allclose(b, a, rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("kw", [dict(), dict(angle_mode=S.ANGLE_PER_TOKEN),
                                dict(decay_mode=S.DECAY_PER_HEAD)])
def test_zoh_gradients_match_central_differences(kw):
    sh = tiny(batch=1, seqlen=10, nheads=2, headdim=2, n_real=3, n_pairs=2, two_endpoint=0,
              discretization=S.DISC_ZOH, **kw)
    inp = inputs(sh, seed=33)
    g = oracle.scan_bwd(sh, inp, inp["dy"])
    eps = 1e-6
    rng = np.random.default_rng(3)
    for key, gkey in (("dt", "ddt"), ("A_log", "dA_log"), ("theta", "dtheta"), ("Bm", "dBm"),
                      ("x", "dx"), ("Cm", "dCm"), ("h0", "dh0")):
        flat = inp[key].reshape(-1)
        for i in rng.choice(flat.size, size=min(flat.size, 12), replace=False):
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(sh, inp)
            flat[i] = old - eps
            lm = _loss(sh, inp)
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            an = g[gkey].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (key, i, fd, an)
