"""Pins of the oracle's dense-output save points (steps that do not stop at the
save times; the state there read off the dense output of the step that
contains it -- Tsit5's own continuous extension, the cubic Hermite interpolant
for the Rosenbrock methods -- the loss and its derivative through it).

* The continuous extension's coefficients: every fourth-order condition holds
  for all theta, b(1) = b, b'(0) = e_1 and b'(1) = e_7 (exact rationals of the
  stored doubles); the weights as formed equal the polynomials.
* Closed form on u' = p u: with z = p h a step multiplies the state by R(z);
  the Tsit5 dense output at theta is u_s (1 + z b(theta)^T (I - z A)^-1 1)
  (A the 7-stage matrix with b as its last row), the Hermite one
  (H00 + z H10) u_s + (H01 + z H11) u_{s+1}, u_s = u0 prod R; their
  derivatives by p and u0 follow in exact rationals (theta is data).
* Order: one step of Lorenz read at interior theta against DOP853; the local
  error falls as h^5 (fourth-order weights).
* Accuracy: Lorenz at a tight tolerance against scipy's DOP853; the test
  equation against exp(p t).
* Invariants: the dense adaptive solve equals the replay of the dense record
  bit for bit; theta in (0, 1]; the steps before a save point plus theta times
  its step reach the save time; the dense output at theta = 1 is the step's end.
* Two derivative routes (tape and dual numbers) and fixed-mesh differences.
"""
from fractions import Fraction as Fr

import numpy as np
import pytest
from scipy.integrate import solve_ivp

import oracle
import workloads as W
from test_oracle_method import _R_any, _kappa

EPS = np.finfo(np.float64).eps


def _R_dR(method, z):
    return _R_any(method, z)


def _weights(th):
    """H00, H01, H10, H11 of the cubic Hermite basis, exact."""
    th = Fr(th)
    return 1 - th * th * (3 - 2 * th), th * th * (3 - 2 * th), th * (1 - th) ** 2, -th * th * (1 - th)


def _tsit5_exact():
    """c, the 7 x 7 stage matrix (last row b) and the extension's r[7][4], as
    exact rationals of the oracle's doubles."""
    c, A6, _ = oracle.tsit5_tableau()
    A = [[Fr(float(A6[i, j])) if j < 6 else Fr(0) for j in range(7)] for i in range(7)]
    r = oracle.tsit5_dense_coeffs()
    return [Fr(float(x)) for x in c], A, [[Fr(float(x)) for x in row] for row in r]


def _b_theta(r, th):
    return [sum(r[i][m] * th ** (m + 1) for m in range(4)) for i in range(7)]


def _tsit5_D(A, bth, z):
    """(D, D') of D(z) = 1 + z b(theta)^T (I - z A)^-1 1; A strictly lower
    triangular, so (I - z A)^-1 1 = sum_k z^k A^k 1 (k <= 6)."""
    v = [Fr(1)] * 7
    D, dD = Fr(1), Fr(0)
    for k in range(7):
        t = sum(bth[i] * v[i] for i in range(7))
        D += z ** (k + 1) * t
        dD += (k + 1) * z ** k * t
        v = [sum(A[i][j] * v[j] for j in range(7)) for i in range(7)]
    return D, dD


def _trees(c, A):
    """(Phi(t), order, gamma(t)) of the eight trees of order <= 4."""
    def mv(v):
        return [sum(A[i][j] * v[j] for j in range(7)) for i in range(7)]
    one = [Fr(1)] * 7
    c2 = [x * x for x in c]
    Ac = mv(c)
    return [(one, 1, 1), (c, 2, 2), (c2, 3, 3), (Ac, 3, 6), ([x ** 3 for x in c], 4, 4),
            ([c[i] * Ac[i] for i in range(7)], 4, 8), (mv(c2), 4, 12), (mv(Ac), 4, 24)]


def test_tsit5_extension_order_conditions():
    c, A, r = _tsit5_exact()
    for phi, order, gamma in _trees(c, A):
        for m in range(1, 5):  # coefficient of theta^m of sum_i b_i(theta) Phi_i
            got = sum(r[i][m - 1] * phi[i] for i in range(7))
            want = Fr(1, gamma) if m == order else Fr(0)
            mag = sum(abs(r[i][m - 1] * phi[i]) for i in range(7))
            assert abs(float(got - want)) <= 4 * EPS * max(float(mag), 1.0), (order, gamma, m)
    b = A[6]
    for i in range(7):
        assert abs(float(sum(r[i]) - b[i])) <= 4 * EPS * sum(abs(float(x)) for x in r[i]), i  # b(1) = b
        slope1 = sum((m + 1) * r[i][m] for m in range(4))
        assert abs(float(slope1 - (1 if i == 6 else 0))) <= 8 * EPS * 4 * sum(abs(float(x)) for x in r[i]), i
        assert r[i][0] == (1 if i == 0 else 0)  # b'(0) = e_1


@pytest.mark.parametrize("dtype", ["f64", "f32"])
def test_tsit5_weights_as_formed(dtype):
    _, _, r = _tsit5_exact()
    eps = EPS if dtype == "f64" else float(np.finfo(np.float32).eps)
    for th in [0.03125, 0.1, 0.25, 0.5, 0.7, 0.9, 0.999]:
        thd = float(np.float32(th)) if dtype == "f32" else th
        exact = _b_theta([[Fr(float(np.float32(x))) if dtype == "f32" else x for x in row] for row in r], Fr(thd))
        got = oracle.tsit5_dense_weights(thd, dtype)
        for i in range(7):
            scale = sum(abs(float(r[i][m])) * thd ** (m + 1) for m in range(4))
            assert abs(got[i] - float(exact[i])) <= 6 * eps * scale, (th, i)


def _lorenz_rhs(t, u, s, r, b):
    return [s * (u[1] - u[0]), u[0] * (r - u[2]) - u[1], u[0] * u[1] - b * u[2]]


def test_tsit5_dense_local_order():
    """One Tsit5 step from a point of a Lorenz trajectory, read at interior
    theta: the error against DOP853 at 1e-13 falls as h^5."""
    prob = W.lorenz_small(1)
    u0 = prob.u0[:, 0].copy()
    ref0 = solve_ivp(_lorenz_rhs, (0.0, 0.3), u0, method="DOP853", rtol=1e-13, atol=1e-13, args=tuple(prob.p[:, 0]))
    start = ref0.y[:, -1]
    thetas = [0.3, 0.55, 0.8]
    errs = []
    for h in [0.04, 0.02, 0.01]:
        q = prob.subset(np.arange(1))
        q.u0 = start[:, None].copy()
        q.tsave = np.array([th * h for th in thetas])
        mesh = oracle.Mesh(np.array([[h]]), np.array([1], np.int32), np.ones((1, 3), np.int32),
                           np.zeros(1, np.int32), np.zeros(1, np.int32), np.array([thetas]))
        _, us = oracle.replay(q, mesh)
        ref = solve_ivp(_lorenz_rhs, (0.0, h), start, method="DOP853", rtol=1e-13, atol=1e-13,
                        t_eval=[th * h for th in thetas], args=tuple(prob.p[:, 0]))
        errs.append(np.abs(us[:, :, 0].T - ref.y).max())
    rates = np.log2(np.array(errs[:-1]) / np.array(errs[1:]))
    assert (rates >= 4.5).all(), (errs, rates)


@pytest.mark.parametrize("method,lams", [("tsit5", [0.5, 3.0, 12.0]), ("ros2", [0.5, 50.0, 400.0]),
                                         ("ros3", [0.5, 50.0, 400.0])])
def test_closed_form_on_the_test_equation(method, lams):
    prob = W.scalar_linear([-l for l in lams], t1=2.0, method=method)
    prob.tsave = np.array([0.2345, 0.777, 1.3, 2.0])
    prob.rtol = prob.atol = 1e-7 if method == "tsit5" else 1e-4
    mesh = oracle.record(prob, 20000, dense=True)
    assert (mesh.status == 0).all()
    _, us = oracle.replay(prob, mesh)
    S = oracle.sens(prob, mesh)  # [nsave][1][2][n]: columns (p, u0)
    tab = _tsit5_exact() if method == "tsit5" else None
    for i, lam in enumerate(lams):
        p = Fr(-lam)
        hs = [Fr(float(x)) for x in mesh.h[i, : mesh.nsteps[i]]]
        u, du, s = Fr(1), Fr(0), 0  # u_s and d u_s / dp
        for k, sidx in enumerate(mesh.save_idx[i]):
            while s < sidx - 1:
                r, dr = _R_dR(method, p * hs[s])
                du = du * r + u * hs[s] * dr
                u *= r
                s += 1
            h = hs[sidx - 1]
            r, dr = _R_dR(method, p * h)
            un, dun = u * r, du * r + u * h * dr
            z = p * h
            if method == "tsit5":  # u(theta) = D(z) u_s
                D, dD = _tsit5_D(tab[1], _b_theta(tab[2], Fr(float(mesh.theta[i, k]))), z)
                ut = D * u                                        # du0 of it: D R^s (u0 = 1)
                dut = h * dD * u + D * du
            else:
                H00, H01, H10, H11 = _weights(float(mesh.theta[i, k]))
                a, b = H00 + z * H10, H01 + z * H11
                ut = a * u + b * un                               # du0 of it: a R^s + b R^{s+1} (u0 = 1)
                dut = h * H10 * u + a * du + h * H11 * un + b * dun
            tol = 4 * sidx * EPS * _kappa(method, -lam, mesh.h[i, :sidx]) * (32 if method == "tsit5" else 8)
            assert abs(us[k, 0, i] - float(ut)) <= tol * abs(float(ut)), (method, lam, k)
            assert abs(S[k, 0, 1, i] - float(ut)) <= tol * abs(float(ut))  # d/du0 with u0 = 1
            assert abs(S[k, 0, 0, i] - float(dut)) <= tol * abs(float(dut)), (method, lam, k)


def test_test_equation_accuracy():
    lams = [0.5, 2.0, 6.0]
    prob = W.scalar_linear([-l for l in lams], t1=1.0)
    prob.tsave = np.array([0.1234, 0.5, 0.8765, 1.0])
    prob.rtol = prob.atol = 1e-8
    us, _, st = oracle.solve_adaptive(prob, 200000, dense=True)
    assert (st == 0).all()
    assert np.abs(us[:, 0, :] - np.exp(-np.outer(prob.tsave, lams))).max() <= 50 * prob.rtol


def _lorenz(t, u, s, r, b):
    return [s * (u[1] - u[0]), u[0] * (r - u[2]) - u[1], u[0] * u[1] - b * u[2]]


def test_lorenz_against_dop853():
    prob = W.lorenz_small(4)
    prob.rtol = prob.atol = 1e-10
    prob.tsave = np.array([0.137, 0.5, 0.911, 1.0])
    us, _, st = oracle.solve_adaptive(prob, 4000, dense=True)
    assert (st == 0).all()
    for i in range(prob.n):
        ref = solve_ivp(_lorenz, (0.0, 1.0), prob.u0[:, i], method="DOP853", rtol=1e-13, atol=1e-13,
                        t_eval=prob.tsave, args=tuple(prob.p[:, i]))
        err = np.abs(us[:, :, i].T - ref.y).max() / np.abs(ref.y).max()
        assert err <= 1e-7, err


@pytest.mark.parametrize("name", ["lorenz_1m", "robertson"])
def test_invariants(name):
    prob = W.by_name(name, n=5)
    smax = 20000 if name == "robertson" else 2048
    mesh = oracle.record(prob, smax, dense=True)
    assert (mesh.status == 0).all()
    assert ((mesh.theta > 0) & (mesh.theta <= 1)).all()
    us, ns, st = oracle.solve_adaptive(prob, smax, dense=True)
    _, ur = oracle.replay(prob, mesh)
    assert np.array_equal(ns, mesh.nsteps) and np.array_equal(us, ur)
    for i in range(prob.n):
        t = np.concatenate([[0.0], np.cumsum(mesh.h[i, : mesh.nsteps[i]])]) + prob.t0
        for k, ts in enumerate(prob.tsave):
            s = mesh.save_idx[i, k]
            assert abs(t[s - 1] + mesh.theta[i, k] * mesh.h[i, s - 1] - ts) <= 4 * s * EPS * abs(prob.t1)
    # theta = 1 reads the step's end: the same mesh with the save points moved
    # to the ends of their steps replays to the states there
    land = oracle.Mesh(mesh.h, mesh.nsteps, mesh.save_idx, mesh.status, mesh.nreject, np.ones_like(mesh.theta))
    _, ul = oracle.replay(prob, land)
    _, un = oracle.replay(prob, oracle.Mesh(mesh.h, mesh.nsteps, mesh.save_idx, mesh.status, mesh.nreject))
    assert np.array_equal(ul, un)


@pytest.mark.parametrize("name", ["lorenz_1m", "robertson"])
def test_tape_equals_dual(name):
    prob = W.by_name(name, n=4)
    mesh = oracle.record(prob, 20000 if name == "robertson" else 2048, dense=True)
    a, b = oracle.grad(prob, mesh, "tape"), oracle.grad(prob, mesh, "dual")
    S = mesh.nsteps.max()
    for key in ("dp", "du0"):
        e = np.abs(a[key] - b[key]).max(0) / np.abs(b[key]).max(0)
        assert e.max() <= 4 * max(1e-13, EPS * S), (key, e.max())


def test_fixed_mesh_differences():
    prob = W.lorenz_small(3)
    prob.tsave = np.array([0.33, 0.71, 1.0])
    prob.target = np.zeros((3, 3, prob.n))
    mesh = oracle.record(prob, 512, dense=True)
    g = oracle.grad(prob, mesh, "tape_wide")
    for j in range(6):
        col = np.zeros((3, prob.n))
        col[j % 3] = 1.0

        def L(e):
            q = prob.subset(np.arange(prob.n))
            if j < 3:
                q.p = q.p + e * col
            else:
                q.u0 = q.u0 + e * col
            return oracle.replay(q, mesh)[0]

        e = 1e-4 if j >= 3 else 1e-3
        cd = lambda e: (L(e) - L(-e)) / (2 * e)
        fd = (4 * cd(e / 2) - cd(e)) / 3
        ref = (g["dp"] if j < 3 else g["du0"])[j % 3]
        assert np.abs(fd - ref).max() <= 1e-7 * np.abs(ref).max(), j
