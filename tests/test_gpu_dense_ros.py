"""GPU <-> oracle parity for dense-output save points with the Rosenbrock
methods (ROS2 and ROS3) on the d = 3 systems: steps stop only at t1, and the
state at a save time inside a step is the cubic Hermite interpolant on the
step's end states and their slopes (two evaluations of f).  Checked: the
dense record (step counts, step sizes, positions theta), the replay and the
adaptive forward-only solve, and the gradient through the interpolant."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import (TOL, dev, ensemble, loss_args, mesh_by_trajectory, mesh_from_oracle, mesh_rel_err, parity,
                      sens_parity, theta_by_trajectory)

pytestmark = pytest.mark.gpu


def _robertson(n, method, dtype="f64"):
    """The robertson ensemble with seven save times spread over [0, 1e5] (none
    of which a dense record lands on) and a linear loss at each."""
    prob = W.robertson(n)
    prob.method = method
    prob.tsave = np.array([0.37, 3.7, 37.0, 370.0, 3700.0, 37000.0, 1e5])
    prob.weight = np.random.default_rng(21).uniform(0.0, 1.0, (len(prob.tsave), 3, n))
    return prob.as_dtype(dtype)


def _lorenz(n, method, dtype="f64"):
    """lorenz_1m's ensemble over t in [0, 0.6] with three interior save times
    (ROS2 on this non-stiff, chaotic system takes ~10^4 steps per time unit
    at rtol = atol = 1e-6)."""
    prob = W.lorenz_1m(n, dtype=dtype)
    prob.method = method
    prob.t1 = 0.6
    prob.tsave = np.array([0.12345, 0.3141592653589793, 0.47, 0.6])
    prob.target = prob.target[: len(prob.tsave)].copy()
    return prob


CASES = [("robertson", "ros2"), ("robertson", "ros3"), ("lorenz", "ros2"), ("lorenz", "ros3")]
SMAX = {("robertson", "ros2"): 20000, ("robertson", "ros3"): 4096, ("lorenz", "ros2"): 16384,
        ("lorenz", "ros3"): 2048}


def _make(system, method, n, dtype="f64"):
    return _robertson(n, method, dtype) if system == "robertson" else _lorenz(n, method, dtype)


@pytest.fixture(scope="module", params=CASES, ids=lambda c: f"{c[0]}-{c[1]}")
def case(request):
    system, method = request.param
    prob = _make(system, method, 600)
    om = oracle.record(prob, SMAX[request.param], dense=True)
    assert (om.status == 0).all() and (om.theta[:, :-1] < 1).all()
    return prob, om, SMAX[request.param]


def test_dense_record_matches_oracle(case):
    prob, om, smax = case
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, smax, len(prob.tsave), prob.dtype, dev(), dense=True)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert (st == 0).all()
    assert np.array_equal(ns, om.nsteps) and np.array_equal(si, om.save_idx)
    assert mesh_rel_err(h, om.h, ns) <= 1e-10
    assert np.abs(theta_by_trajectory(mesh) - om.theta).max() <= 1e-10
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, smax, dense=True)
    torch.cuda.synchronize()
    assert np.array_equal(nsteps.cpu().numpy(), om.nsteps)


def test_dense_replay_and_adaptive_solve(case):
    prob, om, smax = case
    _, ur = oracle.replay(prob, om)
    u = gs.gs_solve(ensemble(prob), mesh_from_oracle(om, "f64")).cpu().numpy()
    scale = np.abs(ur).max(axis=(0, 1))
    assert (np.abs(u - ur).max(axis=(0, 1)) <= 1e-14 * scale).all()
    ua, na, sa = gs.gs_solve_adaptive(ensemble(prob), prob.rtol, prob.atol, smax, dense=True)
    torch.cuda.synchronize()
    assert (sa == 0).all() and np.array_equal(na.cpu().numpy(), om.nsteps)
    assert (np.abs(ua.cpu().numpy() - ur).max(axis=(0, 1)) <= 1e-10 * scale).all()


@pytest.mark.parametrize("perm", [False, True])
def test_dense_gradient_on_oracle_mesh(case, perm):
    prob, om, _ = case
    order = np.random.default_rng(4).permutation(prob.n) if perm else None
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f64", order), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om)
    loss, _ = oracle.replay(prob, om)
    assert np.abs(out.loss.cpu().numpy() - loss).max() <= 1e-14 * np.abs(loss).max()


@pytest.mark.parametrize("system,method", CASES)
def test_dense_gradient_fp32(system, method):
    prob = _make(system, method, 300, "f32")
    om = oracle.record(prob, SMAX[(system, method)], dense=True)
    ok = om.status == 0
    assert ok.mean() > 0.9
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f32"), **loss_args(prob))
    torch.cuda.synchronize()
    sub = np.flatnonzero(ok)
    parity(gs.GradOut(out.loss[sub], out.dp[:, sub], out.du0[:, sub], None), prob.subset(sub),
           _sub_mesh(om, sub), tol=TOL["f32"])


def test_dense_sensitivities(case):
    """Forward sensitivities on the dense mesh: at each save point the tangent
    of the Hermite interpolant (f and its Jacobian-vector product at both
    step ends), against the oracle's wide-tape matrices, and the loss
    gradient by forward mode against the adjoint's parity."""
    prob, om, _ = case
    idx = np.arange(40)
    sub, osub = prob.subset(idx), _sub_mesh(om, idx)
    out, S = gs.gs_sens(ensemble(sub), mesh_from_oracle(osub, "f64"), **loss_args(sub))
    torch.cuda.synchronize()
    sens_parity(S.double().cpu().numpy(), sub, osub, TOL["f64"])
    parity(out, sub, osub)
    loss, _ = oracle.replay(sub, osub)
    assert np.abs(out.loss.cpu().numpy() - loss).max() <= 1e-14 * np.abs(loss).max()


def _sub_mesh(om, idx):
    return oracle.Mesh(om.h[idx], om.nsteps[idx], om.save_idx[idx], om.status[idx], om.nreject[idx],
                       None if om.theta is None else om.theta[idx])


def test_dense_robertson_full_size_sampled():
    """The robertson ensemble at its full 65,536 with ROS3 and the seven
    interior save times, in the launch configuration of the product path; the
    oracle checks a sample."""
    prob = _robertson(65536, "ros3")
    ens = ensemble(prob)
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 4096, dense=True)
    smax = int(nsteps.max().item())
    mesh = gs.new_mesh(prob.n, smax, len(prob.tsave), "f64", dev(), dense=True)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    assert (mesh.status == 0).all() and torch.isfinite(out.dp).all()
    ns_all = nsteps.cpu().numpy()
    rng = np.random.default_rng(15)
    idx = np.unique(np.concatenate([rng.choice(prob.n, 192, replace=False), np.argsort(ns_all)[-16:]]))
    sub = prob.subset(idx)
    om = oracle.record(sub, 4096, dense=True)
    assert np.array_equal(ns_all[idx], om.nsteps)
    ti = torch.tensor(idx, device=dev())
    parity(gs.GradOut(out.loss[ti], out.dp[:, ti], out.du0[:, ti], None), sub, om)
