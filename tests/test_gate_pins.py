"""Pins of the oracle's output gate (y_g = y * silu(z)) against closed forms,
symmetry and central differences; none of them calls the function under test
for its expected value."""
import math

import numpy as np

import oracle


def test_gate_closed_forms():
    z = np.array([-30.0, -2.0, -0.5, 0.0, 0.5, 2.0, 30.0])
    y = np.array([1.5, -2.0, 3.0, 7.0, -1.0, 0.25, 2.0])
    silu = np.array([v / (1.0 + math.exp(-v)) for v in z])
    assert np.allclose(oracle.gate_fwd(y, z), y * silu, rtol=1e-13, atol=1e-300)
    assert oracle.gate_fwd(np.array([3.0]), np.array([0.0]))[0] == 0.0   # silu(0) = 0
    # silu(z) - silu(-z) = z
    zz = np.linspace(-8, 8, 33)
    one = np.ones_like(zz)
    assert np.allclose(oracle.gate_fwd(one, zz) - oracle.gate_fwd(one, -zz), zz, atol=1e-13)


def test_gate_derivative_at_zero():
    # d silu / dz at 0 is 1/2, so dz = dyg * y / 2 there; dy = dyg * silu(0) = 0
    dy, dz = oracle.gate_bwd(np.array([4.0]), np.array([0.0]), np.array([3.0]))
    assert dy[0] == 0.0 and abs(dz[0] - 6.0) < 1e-15


def test_gate_gradients_match_central_differences():
    g = np.random.default_rng(3)
    y, z, dyg = g.standard_normal((3, 40))
    dy, dz = oracle.gate_bwd(y, z, dyg)
    h = 1e-6
    loss = lambda yy, zz: float(np.sum(dyg * oracle.gate_fwd(yy, zz)))  # noqa: E731
    for i in range(0, 40, 7):
        e = np.zeros(40)
        e[i] = h
        ny = (loss(y + e, z) - loss(y - e, z)) / (2 * h)
        nz = (loss(y, z + e) - loss(y, z - e)) / (2 * h)
        assert abs(ny - dy[i]) <= 1e-7 * max(1.0, abs(ny))
        assert abs(nz - dz[i]) <= 1e-7 * max(1.0, abs(nz))
