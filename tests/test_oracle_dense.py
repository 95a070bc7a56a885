"""Pins of the oracle's dense-output save points (steps that do not stop at the
save times; the state there read off the cubic Hermite interpolant of the step
that contains it, the loss and its derivative through that interpolant).

* Closed form on u' = p u: with z = p h, a step multiplies the state by R(z)
  and f(u) = p u, so the interpolated state at theta inside step s is
  (H00 + z H10) u_s + (H01 + z H11) u_{s+1},  u_s = u0 prod R,
  and its derivatives by p and u0 follow in exact rationals (theta is data).
* Accuracy: Lorenz at a tight tolerance against scipy's DOP853; the test
  equation against exp(p t).
* Invariants: the dense adaptive solve equals the replay of the dense record
  bit for bit; theta in (0, 1]; the steps before a save point plus theta times
  its step reach the save time; the interpolant at theta = 1 is the step's end.
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
            H00, H01, H10, H11 = _weights(float(mesh.theta[i, k]))
            z = p * h
            a, b = H00 + z * H10, H01 + z * H11
            ut = a * u + b * un                                   # du0 of it: a R^s + b R^{s+1} (u0 = 1)
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
