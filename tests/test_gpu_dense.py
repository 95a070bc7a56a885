"""GPU <-> oracle parity for dense-output save points (steps that do not stop
at the save times; the state there read off Tsit5's continuous extension):
the dense record (step counts, step sizes and save-point positions), the
replay and the adaptive forward-only solve, and the gradient through the
interpolant, on Lorenz with Tsit5 (ten save points strictly inside steps)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import (TOL, dev, ensemble, loss_args, mesh_by_trajectory, mesh_from_oracle, mesh_rel_err, parity,
                      sens_parity, theta_by_trajectory)

pytestmark = pytest.mark.gpu


def _prob(n, dtype="f64"):
    """lorenz_1m's ensemble with save times that no landing record would hit."""
    prob = W.lorenz_1m(n, dtype=dtype)
    prob.tsave = prob.tsave - 0.3141592653589793
    prob.tsave[-1] = prob.t1
    return prob


def _record_gpu(prob, smax):
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, smax, len(prob.tsave), prob.dtype, dev(), dense=True)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    return ens, mesh


@pytest.fixture(scope="module")
def case():
    prob = _prob(3000)
    om = oracle.record(prob, 1024, dense=True)
    assert (om.status == 0).all() and (om.theta[:, :-1] < 1).all()
    return prob, om


def test_dense_record_matches_oracle(case):
    prob, om = case
    ens, mesh = _record_gpu(prob, 1024)
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert (st == 0).all()
    assert np.array_equal(ns, om.nsteps) and np.array_equal(si, om.save_idx)
    assert mesh_rel_err(h, om.h, ns) <= 1e-10
    th = theta_by_trajectory(mesh)
    assert np.abs(th - om.theta).max() <= 1e-10
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 1024, dense=True)
    torch.cuda.synchronize()
    assert np.array_equal(nsteps.cpu().numpy(), om.nsteps)


def test_dense_replay_and_adaptive_solve(case):
    prob, om = case
    _, ur = oracle.replay(prob, om)
    u = gs.gs_solve(ensemble(prob), mesh_from_oracle(om, "f64")).cpu().numpy()
    assert np.abs(u - ur).max() <= 1e-14 * np.abs(ur).max()
    ua, na, sa = gs.gs_solve_adaptive(ensemble(prob), prob.rtol, prob.atol, 1024, dense=True)
    torch.cuda.synchronize()
    assert (sa == 0).all() and np.array_equal(na.cpu().numpy(), om.nsteps)
    e = np.abs(ua.cpu().numpy() - ur).max(axis=(0, 1)) / np.abs(ur).max(axis=(0, 1))
    assert e.max() <= 1e-10


@pytest.mark.parametrize("perm", [False, True])
def test_dense_gradient_on_oracle_mesh(case, perm):
    prob, om = case
    order = np.random.default_rng(4).permutation(prob.n) if perm else None
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f64", order), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om)
    loss, _ = oracle.replay(prob, om)
    assert np.abs(out.loss.cpu().numpy() - loss).max() <= 1e-14 * np.abs(loss).max()


def test_dense_gradient_fp32():
    prob = _prob(1000, "f32")
    om = oracle.record(prob, 1024, dense=True)
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f32"), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om, tol=TOL["f32"])


def test_dense_linear_loss_and_own_mesh(case):
    """The linear loss through the interpolant, on the GPU's own dense record."""
    prob, om = case
    prob = prob.subset(np.arange(prob.n))
    prob.loss, prob.target = "linear", None
    prob.weight = np.random.default_rng(5).uniform(0, 1, (10, 3, prob.n))
    ens, mesh = _record_gpu(prob, 1024)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om)


def test_dense_sensitivities(case):
    """Forward sensitivities on the dense mesh: at each save point the tangent
    of the continuous extension, against the oracle's dual numbers on the same
    mesh, and the loss gradient equal to the adjoint's."""
    prob, om = case
    sub = prob.subset(np.arange(256))
    osub = oracle.Mesh(om.h[:256], om.nsteps[:256], om.save_idx[:256], om.status[:256], om.nreject[:256],
                       om.theta[:256])
    out, S = gs.gs_sens(ensemble(sub), mesh_from_oracle(osub, "f64"), **loss_args(sub))
    torch.cuda.synchronize()
    sens_parity(S.double().cpu().numpy(), sub, osub, TOL["f64"])
    parity(out, sub, osub)
    loss, _ = oracle.replay(sub, osub)
    assert np.abs(out.loss.cpu().numpy() - loss).max() <= 1e-14 * np.abs(loss).max()


def test_dense_several_save_points_per_step():
    """Save times closer than the steps (48 in t in [0.01, 0.5] on Lorenz at
    rtol = atol = 1e-5): several fall inside one step, each read off that
    step's continuous extension. Record, adaptive solve, replay, gradient and
    forward sensitivities against the oracle."""
    prob = W.lorenz_small(300)
    prob.rtol = prob.atol = 1e-5
    prob.t1 = 0.5
    prob.tsave = np.linspace(0.01, 0.5, 48)
    prob.target = np.random.default_rng(8).normal(0.0, 1.0, (48, 3, prob.n))
    om = oracle.record(prob, 512, dense=True)
    assert (om.status == 0).all()
    assert (np.diff(om.save_idx, axis=1) == 0).any()  # save points sharing a step
    ens, mesh = _record_gpu(prob, 512)
    h, ns, si, st, _ = mesh_by_trajectory(mesh)
    assert np.array_equal(ns, om.nsteps) and np.array_equal(si, om.save_idx)
    assert np.abs(theta_by_trajectory(mesh) - om.theta).max() <= 1e-10
    _, ur = oracle.replay(prob, om)
    u = gs.gs_solve(ens, mesh_from_oracle(om, "f64")).cpu().numpy()
    assert np.abs(u - ur).max() <= 1e-14 * np.abs(ur).max()
    ua, na, sa = gs.gs_solve_adaptive(ens, prob.rtol, prob.atol, 512, dense=True)
    uo, no, so = oracle.solve_adaptive(prob, 512, dense=True)
    assert np.array_equal(ua.cpu().numpy(), uo)  # the same arithmetic: bitwise
    out = gs.gs_grad(ens, mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om)
    sub = prob.subset(np.arange(64))
    osub = oracle.Mesh(om.h[:64], om.nsteps[:64], om.save_idx[:64], om.status[:64], om.nreject[:64],
                       om.theta[:64])
    sout, S = gs.gs_sens(ensemble(sub), mesh_from_oracle(osub, "f64"), **loss_args(sub))
    torch.cuda.synchronize()
    sens_parity(S.double().cpu().numpy(), sub, osub, TOL["f64"])


def test_dense_unsupported_paths(case):
    k8 = W.kin8(4)  # dense records are built for the d = 3 systems
    with pytest.raises(gs.gradsolve.GradsolveError):
        gs.gs_count(ensemble(k8), k8.rtol, k8.atol, 100, dense=True)


def test_full_size_sampled():
    """2**20 trajectories, dense record + gradient in the benchmark's launch
    configuration; the oracle checks a sample (random + the longest chains)."""
    prob = _prob(1 << 20)
    ens = ensemble(prob)
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 2048, dense=True)
    smax = int(nsteps.max().item())
    mesh = gs.new_mesh(prob.n, smax, 10, "f64", dev(), dense=True)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    assert (mesh.status == 0).all() and torch.isfinite(out.dp).all()
    ns_all = nsteps.cpu().numpy()
    rng = np.random.default_rng(14)
    idx = np.unique(np.concatenate([rng.choice(prob.n, 256, replace=False), np.argsort(ns_all)[-16:]]))
    sub = prob.subset(idx)
    om = oracle.record(sub, 2048, dense=True)
    assert np.array_equal(ns_all[idx], om.nsteps)
    ti = torch.tensor(idx, device=dev())
    parity(gs.GradOut(out.loss[ti], out.dp[:, ti], out.du0[:, ti], None), sub, om)
