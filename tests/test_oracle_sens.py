"""Pins of the oracle's forward sensitivities d u(t_k) / d (p, u0) of the
fixed-step replay (the in-kernel forward-sensitivity route; GRADSOLVE
review: the derivative is that of the replay with the mesh held fixed).

* Closed form: on u' = p u a step multiplies the state by R(p h), so
  u_k = u0 prod R(z_s) and, with z_s = p h_s,
  du_k/du0 = prod R(z_s),  du_k/dp = u_k sum_s h_s R'(z_s) / R(z_s),
  over the recorded steps up to the save point, in exact rationals.
* Second route: the chain rule through the sensitivities,
  sum_k (d l_k / d u_k)^T S_k, equals the reverse-mode tape gradient.
* Fixed-mesh central differences with Richardson extrapolation.
* A trajectory whose record failed gets NaN.
"""
from fractions import Fraction as Fr

import numpy as np
import pytest

import oracle
import workloads as W
from test_oracle_method import _R_any, _kappa

EPS = np.finfo(np.float64).eps


_R_dR = _R_any


@pytest.mark.parametrize("method,lams", [("tsit5", [0.5, 3.0, 12.0]), ("ros2", [0.5, 50.0, 400.0]),
                                         ("ros3", [0.5, 50.0, 400.0])])
def test_closed_form_on_the_test_equation(method, lams):
    prob = W.scalar_linear([-l for l in lams], t1=2.0, method=method)
    prob.tsave = np.array([0.25, 1.0, 2.0])
    prob.rtol = prob.atol = 1e-7 if method == "tsit5" else 1e-4
    mesh = oracle.record(prob, 20000)
    S = oracle.sens(prob, mesh)  # [nsave][1][2][n]: columns (p, u0)
    for i, lam in enumerate(lams):
        hs = mesh.h[i, : mesh.nsteps[i]]
        prod, acc, s = Fr(1), Fr(0), 0
        for k, sidx in enumerate(mesh.save_idx[i]):
            while s < sidx:
                r, dr = _R_dR(method, Fr(-lam) * Fr(float(hs[s])))
                prod *= r
                acc += Fr(float(hs[s])) * dr / r
                s += 1
            tol = sidx * EPS * _kappa(method, -lam, hs[:sidx]) * (32 if method == "tsit5" else 8)
            du0, dp = float(prod), float(prod * acc)
            assert abs(S[k, 0, 1, i] - du0) <= tol * abs(du0), (method, lam, k)
            assert abs(S[k, 0, 0, i] - dp) <= tol * abs(dp), (method, lam, k)


@pytest.mark.parametrize("name", ["lorenz_1m", "robertson"])
def test_chain_rule_equals_tape_gradient(name):
    prob = W.by_name(name, n=5)
    mesh = oracle.record(prob, 20000 if name == "robertson" else 1024)
    S = oracle.sens(prob, mesh)
    _, us = oracle.replay(prob, mesh)
    g = oracle.grad(prob, mesh, mode="tape_wide")
    if prob.loss == "sumsq":
        tg = prob.target if prob.target is not None else 0.0
        dl = 2.0 * (us - tg)
    else:
        dl = prob.weight
    gs = np.einsum("kcn,kcjn->jn", dl, S)
    for j, (ref, part) in enumerate([(g["dp"], slice(0, 3)), (g["du0"], slice(3, 6))]):
        got = gs[part]
        err = np.abs(got - ref).max(axis=0) / np.abs(ref).max(axis=0)
        assert err.max() <= 1e-11, (name, j, err.max())


def test_fixed_mesh_differences():
    prob = W.lorenz_small(3)
    mesh = oracle.record(prob, 256)
    S = oracle.sens(prob, mesh)

    def u_at(dp=None, du=None):
        q = prob.subset(np.arange(prob.n))
        q.p = q.p + (0 if dp is None else dp)
        q.u0 = q.u0 + (0 if du is None else du)
        return oracle.replay(q, mesh)[1]

    for j in range(6):
        col = np.zeros((3, prob.n))
        col[j % 3] = 1.0

        def cd(e):
            kw = ({"dp": e * col} if j < 3 else {"du": e * col})
            kw_m = ({"dp": -e * col} if j < 3 else {"du": -e * col})
            return (u_at(**kw) - u_at(**kw_m)) / (2 * e)

        e = 1e-4 * (10.0 if j < 3 else 1.0)
        fd = (4 * cd(e / 2) - cd(e)) / 3  # Richardson
        err = np.abs(fd - S[:, :, j, :]).max() / np.abs(S[:, :, j, :]).max()
        assert err <= 1e-7, (j, err)


def test_failed_trajectory_is_nan():
    prob = W.lorenz_small(3)
    mesh = oracle.record(prob, 256)
    mesh.status = mesh.status.copy()
    mesh.status[1] = 1
    S = oracle.sens(prob, mesh)
    assert np.isnan(S[..., 1]).all() and np.isfinite(S[..., [0, 2]]).all()
