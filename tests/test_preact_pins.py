"""Pins of the oracle's pre-activations (dt = softplus(z + dt_bias[h]),
lambda = sigmoid(logit)) against closed forms and central differences; none
of them goes through the functions under test for the expected value."""
import math

import numpy as np

import oracle


def test_softplus_inverts_the_bias_recipe():
    # dt_bias = log(expm1(dt0)) puts dt at dt0 for z = 0: log(1 + (e^a - 1)) = a
    dt0 = np.array([1e-3, 3e-3, 1e-2, 5e-2, 1e-1])
    bias = np.array([math.log(math.expm1(v)) for v in dt0])
    dt, _ = oracle.preact_fwd(np.zeros((1, 1, dt0.size)), bias)
    assert np.allclose(dt[0, 0], dt0, rtol=1e-12, atol=0)


def test_softplus_and_sigmoid_closed_forms():
    x = np.linspace(-30, 30, 61)
    dt, lam = oracle.preact_fwd(x[None, None, :], np.zeros(61), x[None, None, :])
    ref_sp = np.array([math.log1p(math.exp(v)) if v < 30 else v + math.log1p(math.exp(-v))
                       for v in x])
    ref_sg = np.array([1.0 / (1.0 + math.exp(-v)) for v in x])
    assert np.allclose(dt[0, 0], ref_sp, rtol=1e-12, atol=1e-300)
    assert np.allclose(lam[0, 0], ref_sg, rtol=1e-12, atol=1e-300)
    assert abs(lam[0, 0, 30] - 0.5) < 1e-15                   # sigmoid(0)
    assert np.allclose(lam[0, 0] + lam[0, 0, ::-1], 1.0)      # sigmoid(-x) = 1 - sigmoid(x)


def test_gradients_match_central_differences():
    rng = np.random.default_rng(3)
    B, L, H = 2, 5, 3
    z = rng.normal(size=(B, L, H))
    bias = rng.normal(size=H)
    logit = rng.normal(size=(B, L, H))
    ddt = rng.normal(size=(B, L, H))
    dlam = rng.normal(size=(B, L, H))

    def loss(z_, b_, g_):
        dt, lam = oracle.preact_fwd(z_, b_, g_)
        return float((ddt * dt).sum() + (dlam * lam).sum())

    dz, dbias, dlogit = oracle.preact_bwd(z, bias, logit, ddt, dlam)
    eps = 1e-6
    for idx in [(0, 0, 0), (1, 4, 2), (0, 2, 1)]:
        zp, zm = z.copy(), z.copy()
        zp[idx] += eps
        zm[idx] -= eps
        fd = (loss(zp, bias, logit) - loss(zm, bias, logit)) / (2 * eps)
        assert abs(fd - dz[idx]) <= 1e-6 * max(1.0, abs(fd))
        gp, gm = logit.copy(), logit.copy()
        gp[idx] += eps
        gm[idx] -= eps
        fd = (loss(z, bias, gp) - loss(z, bias, gm)) / (2 * eps)
        assert abs(fd - dlogit[idx]) <= 1e-6 * max(1.0, abs(fd))
    for h in range(H):
        bp, bm = bias.copy(), bias.copy()
        bp[h] += eps
        bm[h] -= eps
        fd = (loss(z, bp, logit) - loss(z, bm, logit)) / (2 * eps)
        assert abs(fd - dbias[h]) <= 1e-6 * max(1.0, abs(fd))
