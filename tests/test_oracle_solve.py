"""Pins of the oracle's adaptive forward-only solve (GRADSOLVE abstract: the
forward-only solver; the recorder's iteration with the accepted states kept).

* Closed form: on u' = p u every accepted step multiplies the state by the
  method's stability function R(p h), so the state saved at t_k is
  u0 * prod R(p h_s) over the recorded steps up to that save point, evaluated
  here in exact rational arithmetic from the tableau (Tsit5) or from gamma
  (ROS2).  A state saved before its step, at the wrong save index, or with a
  stage dropped misses this by far more than rounding.
* Accuracy: the same states against exp(p t_k) within the tolerance's scale.
* Invariant: the saved states equal, bit for bit, the replay of the mesh the
  recorder keeps for the same problem (one iteration, two outputs).
* Failures: a trajectory that fails has NaN at every save point.
"""
from fractions import Fraction as Fr

import numpy as np
import pytest

import oracle
import workloads as W
from test_oracle_method import _kappa, _poly, _ros2_R, _tsit5_R_coeffs

EPS = np.finfo(np.float64).eps


def _R(method, z):
    if method == "tsit5":
        return _poly(_tsit5_R_coeffs(), z)
    return _ros2_R(z, Fr(oracle.ros2_gamma()))[0]


@pytest.mark.parametrize("method,lams", [("tsit5", [0.5, 3.0, 12.0]), ("ros2", [0.5, 50.0, 400.0])])
def test_saved_states_are_stability_function_products(method, lams):
    prob = W.scalar_linear([-l for l in lams], t1=2.0, method=method)
    prob.tsave = np.array([0.25, 0.5, 1.0, 1.7, 2.0])
    prob.rtol = prob.atol = 1e-7 if method == "tsit5" else 1e-4
    us, ns, st = oracle.solve_adaptive(prob, 20000)
    mesh = oracle.record(prob, 20000)
    assert (st == 0).all() and np.array_equal(ns, mesh.nsteps)
    for i, lam in enumerate(lams):
        hs = mesh.h[i, : ns[i]]
        prod, s = Fr(1), 0
        for k, sidx in enumerate(mesh.save_idx[i]):
            while s < sidx:
                prod *= _R(method, Fr(-lam) * Fr(float(hs[s])))
                s += 1
            # rounding: eps times each step's cancellation factor and weight size
            tol = sidx * EPS * _kappa(method, -lam, hs[:sidx]) * (32 if method == "tsit5" else 8)
            assert abs(us[k, 0, i] - float(prod)) <= tol * abs(float(prod)), (method, lam, k)


@pytest.mark.parametrize("method", ["tsit5", "ros2"])
def test_saved_states_meet_the_tolerance(method):
    lams = [0.5, 2.0, 6.0]
    prob = W.scalar_linear([-l for l in lams], t1=1.0, method=method)
    prob.tsave = np.array([0.1, 0.5, 1.0])
    prob.rtol = prob.atol = 1e-8 if method == "tsit5" else 1e-6
    us, _, st = oracle.solve_adaptive(prob, 200000)
    assert (st == 0).all()
    exact = np.exp(-np.outer(prob.tsave, lams))
    # a controlled local error of rtol per step accumulates to a small multiple
    assert np.abs(us[:, 0, :] - exact).max() <= 50 * prob.rtol


@pytest.mark.parametrize("name", ["lorenz_small", "lorenz_1m", "robertson", "node64"])
def test_saved_states_equal_replay_of_the_record(name):
    prob = W.by_name(name, n=6)
    smax = 20000 if name == "robertson" else 2048
    us, ns, st = oracle.solve_adaptive(prob, smax)
    mesh = oracle.record(prob, smax)
    _, ur = oracle.replay(prob, mesh)
    assert (st == 0).all() and np.array_equal(ns, mesh.nsteps)
    assert np.array_equal(us, ur)


def test_failed_trajectories_are_nan():
    prob = W.lorenz_small(3)
    us, ns, st = oracle.solve_adaptive(prob, 20)  # capacity -> MAXSTEPS
    assert (st == 1).all() and np.isnan(us).all()
    bad = W.lorenz_small(3)
    bad.p = bad.p.copy()
    bad.p[0, 1] = np.nan
    us, ns, st = oracle.solve_adaptive(bad, 512)
    assert list(st) == [0, 3, 0]
    assert np.isnan(us[:, :, 1]).all() and np.isfinite(us[:, :, [0, 2]]).all()
