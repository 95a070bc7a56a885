"""GPU <-> oracle parity for the Rosenbrock path at d = 8 (kin8, 8 x 8 LU in
registers): the recorder (ROS3 and ROS2), the fused replay + reverse sweep,
the replay and the adaptive solve, the forward sensitivities (16 directions),
fp32, failure statuses, and the full 262,144-trajectory ensemble in the
benchmark's launch configuration on a sample."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import (TOL, dev, ensemble, grad_rel_err, loss_args, mesh_by_trajectory, mesh_from_oracle,
                      mesh_rel_err, parity, sens_parity, sens_rel)

pytestmark = pytest.mark.gpu

SMAX3, SMAX2 = 2048, 20000


def _kin8(n=None, method="ros3"):
    prob = W.kin8(n)
    prob.method = method
    return prob


def _multi(prob):
    """Three save points (the loss sums over them)."""
    prob.tsave = np.array([1.0, 10.0, 100.0])
    return prob


@pytest.fixture(scope="module")
def k3():
    prob = _multi(_kin8(200))
    om = oracle.record(prob, SMAX3)
    assert (om.status == 0).all()
    return prob, om, oracle.grad(prob, om)


@pytest.mark.parametrize("method,n,smax", [("ros3", 200, SMAX3), ("ros2", 40, SMAX2)])
def test_record_matches_oracle(method, n, smax):
    prob = _multi(_kin8(n, method))
    om = oracle.record(prob, smax)
    assert (om.status == 0).all()
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, smax, 3, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert (st == 0).all()
    assert np.array_equal(ns, om.nsteps) and np.array_equal(si, om.save_idx)
    assert mesh_rel_err(h, om.h, ns) <= 1e-10
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, smax)
    torch.cuda.synchronize()
    assert np.array_equal(nsteps.cpu().numpy(), om.nsteps)


@pytest.mark.parametrize("perm", [False, True])
def test_ros3_grad(k3, perm):
    prob, om, og = k3
    order = np.random.default_rng(4).permutation(prob.n) if perm else None
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f64", order), **loss_args(prob))
    torch.cuda.synchronize()
    e = grad_rel_err(out, og)
    assert e.max() <= 1e-12, e.max()
    assert np.abs(out.loss.cpu().numpy() - og["loss"]).max() <= 1e-14 * np.abs(og["loss"]).max()


def test_ros2_grad():
    """ROS2 takes ~16,000 steps per trajectory at this tolerance: the
    per-trajectory gate of the parity helper."""
    prob = _multi(_kin8(12, "ros2"))
    om = oracle.record(prob, SMAX2)
    assert (om.status == 0).all()
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om)


def test_solve_and_adaptive_solve(k3):
    prob, om, og = k3
    _, us = oracle.replay(prob, om)
    u = gs.gs_solve(ensemble(prob), mesh_from_oracle(om, "f64")).cpu().numpy()
    assert np.array_equal(u, us)  # the same arithmetic: bitwise
    ua, na, sa = gs.gs_solve_adaptive(ensemble(prob), prob.rtol, prob.atol, SMAX3)
    torch.cuda.synchronize()
    uo, no, so = oracle.solve_adaptive(prob, SMAX3)
    assert (sa.cpu().numpy() == 0).all() and np.array_equal(na.cpu().numpy(), no)
    assert np.array_equal(ua.cpu().numpy(), uo)
    # the three linear invariants hold on the device's solution too
    inv = np.array([[1, 1, 0, 1, 1, 1, 0, 1], [0, 0, 1, 1, 0, 0, 0, 0], [0, 0, 0, 0, 0, 0, 1, 1]], float)
    c0 = inv @ prob.u0
    for k in range(len(prob.tsave)):
        assert np.abs(inv @ ua.cpu().numpy()[k] - c0).max() <= 1e-12


def test_ros3_fp32():
    prob = _multi(_kin8(300)).as_dtype("f32")
    prob.rtol = prob.atol = 1e-5
    om = oracle.record(prob, SMAX3)
    assert (om.status == 0).all()
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, SMAX3, 3, "f32", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert np.array_equal(ns, om.nsteps)
    out = gs.gs_grad(ens, mesh_from_oracle(om, "f32"), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om, tol=TOL["f32"])


@pytest.mark.parametrize("n", [1, 129])
def test_statuses_tiny_and_ragged(n):
    """A NaN rate constant gives NONFINITE, a capacity below some step counts
    MAXSTEPS, both as the oracle's; the failed trajectories get NaN from the
    gradient and the replay, the others match the oracle."""
    prob = _kin8(n)
    prob.p = prob.p.copy()
    prob.p[6, n - 1] = np.nan
    full = oracle.record(prob, SMAX3)
    ok_ns = full.nsteps[full.status == 0]
    smax = int(np.median(ok_ns)) if len(ok_ns) else SMAX3
    om = oracle.record(prob, smax)
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, smax, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    u = gs.gs_solve(ens, mesh)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert np.array_equal(st, om.status)
    assert st[n - 1] == gs.gradsolve.TRAJ_NONFINITE
    bad = st != 0
    assert np.isnan(out.loss.cpu().numpy()[bad]).all() and np.isnan(u.cpu().numpy()[..., bad]).all()
    good = np.flatnonzero(~bad)
    if len(good):
        assert np.isfinite(out.dp.cpu().numpy()[:, good]).all()
        sub = prob.subset(good)
        og = oracle.grad(sub, oracle.Mesh(h[good], ns[good], si[good], st[good], np.zeros(len(good), np.int32)))
        ti = torch.tensor(good, device=dev())
        e = grad_rel_err(gs.GradOut(out.loss[ti], out.dp[:, ti], out.du0[:, ti], None), og)
        assert e.max() <= 1e-12


def test_full_size_sampled():
    """All 262,144 trajectories recorded and differentiated (ROS3) in the
    benchmark's launch configuration; the oracle checks a sample (random +
    longest)."""
    prob = _kin8()
    ens = ensemble(prob)
    nsteps, status = gs.gs_count(ens, prob.rtol, prob.atol, SMAX3)
    smax = int(nsteps.max().item())
    mesh = gs.new_mesh(prob.n, smax, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    assert (mesh.status == 0).all()
    assert torch.isfinite(out.dp).all() and torch.isfinite(out.du0).all()
    ns_all = nsteps.cpu().numpy()
    rng = np.random.default_rng(7)
    idx = np.unique(np.concatenate([rng.choice(prob.n, 56, replace=False), np.argsort(ns_all)[-8:]]))
    sub = prob.subset(idx)
    om = oracle.record(sub, SMAX3)
    order = mesh.order.cpu().numpy()
    inv = np.empty_like(order)
    inv[order] = np.arange(prob.n)
    slots = inv[idx]
    ns = mesh.nsteps.cpu().numpy()[slots]
    assert np.array_equal(ns, om.nsteps)
    hs = mesh.h[:, torch.tensor(slots, device=dev())].cpu().numpy().T
    assert mesh_rel_err(hs, om.h[:, :smax], ns) <= 1e-10
    og = oracle.grad(sub, oracle.Mesh(hs.copy(), ns, mesh.save_idx.cpu().numpy().T[slots], np.zeros(len(idx), np.int32),
                                      np.zeros(len(idx), np.int32)))
    ti = torch.tensor(idx, device=dev())
    e = grad_rel_err(gs.GradOut(out.loss[ti], out.dp[:, ti], out.du0[:, ti], None), og)
    assert e.max() <= 1e-12, e.max()


def test_linear_loss_and_leading_zero_steps():
    """The weighted-linear loss at three save points, and leading zero steps
    (exact identities of both Rosenbrock steps) leave loss and gradient
    bitwise unchanged."""
    prob = _multi(_kin8(64))
    prob.loss = "linear"
    prob.weight = np.random.default_rng(11).uniform(0.0, 1.0, (3, 8, prob.n))
    om = oracle.record(prob, SMAX3)
    og = oracle.grad(prob, om)
    ens = ensemble(prob)
    out = gs.gs_grad(ens, mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    assert grad_rel_err(out, og).max() <= 1e-12
    z = 2
    om2 = oracle.Mesh(np.concatenate([np.zeros((prob.n, z)), om.h], 1), om.nsteps + z, om.save_idx + z,
                      om.status, om.nreject)
    out2 = gs.gs_grad(ens, mesh_from_oracle(om2, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    for a, b in ((out.loss, out2.loss), (out.dp, out2.dp), (out.du0, out2.du0)):
        assert torch.equal(a, b)


def test_ros2_fp32():
    prob = _kin8(100, "ros2").as_dtype("f32")
    prob.rtol = prob.atol = 1e-5
    om = oracle.record(prob, SMAX2)
    assert (om.status == 0).all()
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 2048, 1, "f32", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert np.array_equal(ns, om.nsteps)
    out = gs.gs_grad(ens, mesh_from_oracle(om, "f32"), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om, tol=TOL["f32"])


def test_ros3_sensitivities():
    """Forward sensitivities along the 16 input directions (eight rate
    constants, eight initial states) on the oracle's mesh: per trajectory
    against the wide-tape matrices (the gradient's rule), the loss bitwise
    that of the replay, and the forward-mode gradient at the adjoint's
    parity."""
    prob = _multi(_kin8(40, "ros3"))
    om = oracle.record(prob, SMAX3)
    assert (om.status == 0).all()
    out, S = gs.gs_sens(ensemble(prob), mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    assert S.shape == (3, 8, 16, prob.n)
    sens_parity(S.double().cpu().numpy(), prob, om, TOL["f64"])
    parity(out, prob, om)
    loss, _ = oracle.replay(prob, om)
    assert np.abs(out.loss.cpu().numpy() - loss).max() <= 1e-14 * np.abs(loss).max()


def test_ros2_sensitivities():
    """ROS2 (~16,000 steps per trajectory): the matrices against the oracle's
    dual numbers on the same mesh within eps per step, the forward-mode
    gradient at the adjoint's parity."""
    prob = _multi(_kin8(6, "ros2"))
    om = oracle.record(prob, SMAX2)
    assert (om.status == 0).all()
    out, S = gs.gs_sens(ensemble(prob), mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    tol = max(1e-12, 4 * np.finfo(float).eps * int(om.nsteps.max()))
    e = sens_rel(S.double().cpu().numpy(), oracle.sens(prob, om))
    assert e.max() <= tol, (e.max(), tol)
    parity(out, prob, om)
