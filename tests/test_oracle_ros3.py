"""Pins of the oracle's third-order Rosenbrock method ROS3 (Sandu, Verwer, Blom,
Spee, Carmichael & Potra 1997) against facts fixed outside the oracle.

* The coefficients: brought back to the standard Rosenbrock form (alpha, Gamma,
  b, bhat) in exact rationals, they meet the order conditions of Hairer &
  Wanner (Solving ODEs II, Sec. IV.7, Table 7.1) to order 3, the embedded
  weights to order 2 and not 3; gamma is the root in (1/6, 1/2) of
  x^3 - 3x^2 + 3/2 x - 1/6 (the L-stability condition of a three-stage
  third-order method); the row sums of alpha and Gamma are the published
  alpha_i = (0, gamma, gamma) and gamma_i = (gamma, 0.24291996454816804,
  2.1851380027664058).
* The stability function R(z) = 1 + z b^T (I - z beta)^{-1} 1: R(-inf) = 0,
  |R(iy)| <= 1 on the imaginary axis, R(z) - e^z = O(z^4), and the oracle's
  step on u' = p u equals it to rounding.
* Accuracy: Robertson kinetics at tight tolerances against scipy's Radau at
  1e-12; the adaptive recorder needs far fewer steps than ROS2 at the same
  tolerance on the stiff problem (third order against second).
(The closed-form adjoint on u' = -lambda u, the convergence order, tape = dual
and fixed-mesh differences run in the shared parametrised pins.)
"""
from fractions import Fraction as Fr

import numpy as np
import pytest
from scipy.integrate import solve_ivp

import oracle
import workloads as W
from test_oracle_method import _ros3_R, _ros3_std

EPS = np.finfo(np.float64).eps


def test_gamma_and_reciprocal():
    co = oracle.ros3_coeffs()
    g = co["gamma"]
    assert 1 / 6 < g < 1 / 2
    gf = Fr(g)
    poly = gf**3 - 3 * gf**2 + Fr(3, 2) * gf - Fr(1, 6)
    dpoly = 3 * gf**2 - 6 * gf + Fr(3, 2)
    # the double is within a few ulps of the root
    assert abs(float(poly / dpoly)) <= 2 * EPS * g
    assert abs(Fr(co["inv_gamma"]) * gf - 1) <= EPS


def test_order_conditions():
    alpha, G, beta, b, bh = _ros3_std()
    g = G[0][0]
    a_i = [sum(alpha[i]) for i in range(3)]
    bp = [sum(beta[i][j] for j in range(i)) for i in range(3)]  # beta'_i (strictly lower part)

    def conds(w):
        return [
            sum(w) - 1,
            sum(w[i] * bp[i] for i in range(3)) - (Fr(1, 2) - g),
            sum(w[i] * a_i[i] ** 2 for i in range(3)) - Fr(1, 3),
            sum(w[i] * beta[i][k] * bp[k] for i in range(3) for k in range(i)) - (Fr(1, 6) - g + g * g),
        ]

    c = [abs(float(x)) for x in conds(b)]
    assert max(c) <= 1e-14, c
    ch = [abs(float(x)) for x in conds(bh)]
    assert max(ch[:2]) <= 1e-14, ch        # embedded solution: order 2
    assert min(ch[2:]) >= 1e-3, ch         # ... and not order 3
    # published row sums
    assert [float(x) for x in a_i] == pytest.approx([0.0, float(g), float(g)], abs=1e-15)
    gs = [float(sum(G[i])) for i in range(3)]
    assert gs == pytest.approx([float(g), 0.24291996454816804, 2.1851380027664058], rel=1e-14)


def test_stability_function():
    r_big, _ = _ros3_R(Fr(-10**30))
    assert abs(float(r_big)) < 1e-25                       # L-stable
    for e in (Fr(1, 10**3), Fr(-1, 10**3)):
        r, _ = _ros3_R(e)
        taylor = 1 + e + e * e / 2 + e**3 / 6
        assert abs(float((r - taylor) / e**4)) < 1.0       # order 3
    _, _, beta, b, _ = _ros3_std()
    B = np.array([[float(x) for x in row] for row in beta])
    bv = np.array([float(x) for x in b])
    for y in np.concatenate([np.logspace(-3, 4, 60), -np.logspace(-3, 4, 60)]):
        z = 1j * y
        R = 1 + z * bv @ np.linalg.solve(np.eye(3) - z * B, np.ones(3))
        assert abs(R) <= 1 + 1e-13, (y, abs(R))            # A-stable on the axis


def test_step_matches_stability_function():
    for lam, h in [(0.7, 0.1), (1e3, 0.05), (3.0, 2.0), (1e6, 1.0)]:
        un, err, ok = oracle.step("linear", "ros3", "f64", [1.0], [-lam], h)
        r, _ = _ros3_R(Fr(-lam) * Fr(h))
        assert ok and abs(un[0] - float(r)) <= 16 * EPS * max(1.0, abs(float(r))), (lam, h)


def _robertson(t, y, k1, k2, k3):
    return [-k1 * y[0] + k3 * y[1] * y[2], k1 * y[0] - k3 * y[1] * y[2] - k2 * y[1] ** 2, k2 * y[1] ** 2]


def test_robertson_accuracy_against_radau():
    prob = W.robertson(3)
    prob.method = "ros3"
    prob.rtol, prob.atol = 1e-8, 1e-12
    us, ns, st = oracle.solve_adaptive(prob, 20000)
    assert (st == 0).all()
    for i in range(prob.n):
        ref = solve_ivp(_robertson, (prob.t0, prob.t1), prob.u0[:, i], method="Radau", rtol=1e-12, atol=1e-16,
                        t_eval=prob.tsave, args=tuple(prob.p[:, i]))
        assert ref.success
        got = us[:, :, i].T
        # y1, y3 to a relative 1e-6; y2 (~1e-5 .. 1e-10) to 1e-6 of its scale
        for c in range(3):
            sc = np.abs(ref.y[c]).max()
            assert np.abs(got[c] - ref.y[c]).max() <= 1e-6 * sc, (i, c)


def test_fewer_steps_than_ros2_on_stiff_problem():
    prob = W.robertson(4)
    prob.rtol, prob.atol = 1e-8, 1e-12
    n2 = oracle.record(prob, 200000).nsteps
    prob.method = "ros3"
    m3 = oracle.record(prob, 200000)
    assert (m3.status == 0).all()
    assert (m3.nsteps * 4 < n2).all(), (m3.nsteps, n2)
