"""GPU <-> oracle parity for the third-order Rosenbrock path (ROS3): Robertson
kinetics with the robertson workload's ensemble and loss, Lorenz integrated
with ROS3 (fp64 and fp32), and the full 65,536-trajectory Robertson ensemble
in the benchmark's launch configuration on a sample."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import (TOL, dev, ensemble, grad_rel_err, loss_args, mesh_by_trajectory, mesh_from_oracle,
                      mesh_rel_err, parity, tens)

pytestmark = pytest.mark.gpu


def _rob(n=None):
    prob = W.robertson(n)
    prob.method = "ros3"
    return prob


@pytest.fixture(scope="module")
def rob():
    prob = _rob(300)
    om = oracle.record(prob, 4096)
    og = oracle.grad(prob, om)
    assert (om.status == 0).all()
    return prob, om, og


def test_robertson_record(rob):
    prob, om, og = rob
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 4096, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert (st == 0).all()
    assert np.array_equal(ns, om.nsteps) and np.array_equal(si, om.save_idx)
    assert mesh_rel_err(h, om.h, ns) <= 1e-10
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 4096)
    torch.cuda.synchronize()
    assert np.array_equal(nsteps.cpu().numpy(), om.nsteps)


@pytest.mark.parametrize("perm", [False, True])
def test_robertson_grad(rob, perm):
    prob, om, og = rob
    order = np.random.default_rng(3).permutation(prob.n) if perm else None
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f64", order), **loss_args(prob))
    torch.cuda.synchronize()
    e = grad_rel_err(out, og)
    assert e.max() <= 1e-12, e.max()
    assert np.abs(out.loss.cpu().numpy() - og["loss"]).max() <= 1e-14 * np.abs(og["loss"]).max()


def test_robertson_solve_and_adaptive_solve(rob):
    prob, om, og = rob
    _, us = oracle.replay(prob, om)
    u = gs.gs_solve(ensemble(prob), mesh_from_oracle(om, "f64")).cpu().numpy()
    assert np.abs(u - us).max() <= 1e-14
    ua, na, sa = gs.gs_solve_adaptive(ensemble(prob), prob.rtol, prob.atol, 4096)
    torch.cuda.synchronize()
    uo, no, so = oracle.solve_adaptive(prob, 4096)
    assert (sa.cpu().numpy() == 0).all() and np.array_equal(na.cpu().numpy(), no)
    assert np.array_equal(ua.cpu().numpy(), uo)  # the same arithmetic: bitwise


def test_lorenz_ros3_record_and_grad():
    prob = W.lorenz_small(500)
    prob.method = "ros3"
    prob.rtol = prob.atol = 1e-5
    om = oracle.record(prob, 8192)
    og = oracle.grad(prob, om)
    assert (om.status == 0).all()
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 8192, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert np.array_equal(ns, om.nsteps)
    assert mesh_rel_err(h, om.h, ns) <= 1e-10
    out = gs.gs_grad(ens, mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    assert grad_rel_err(out, og).max() <= 1e-12


def test_lorenz_ros3_grad_fp32():
    prob = W.lorenz_small(400)
    prob.method = "ros3"
    prob.dtype = "f32"
    prob.rtol = prob.atol = 1e-4
    om = oracle.record(prob, 8192)
    assert (om.status == 0).all()
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f32"), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om, tol=TOL["f32"])


def test_robertson_full_size_sampled():
    """All 65,536 trajectories recorded and differentiated in the benchmark's
    launch configuration; the oracle checks a sample (random + longest)."""
    prob = _rob()
    ens = ensemble(prob)
    nsteps, status = gs.gs_count(ens, prob.rtol, prob.atol, 20000)
    smax = int(nsteps.max().item())
    mesh = gs.new_mesh(prob.n, smax, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    assert (mesh.status == 0).all()
    ns_all = nsteps.cpu().numpy()
    rng = np.random.default_rng(6)
    idx = np.unique(np.concatenate([rng.choice(prob.n, 96, replace=False), np.argsort(ns_all)[-8:]]))
    sub = prob.subset(idx)
    om = oracle.record(sub, 20000)
    order = mesh.order.cpu().numpy()
    inv = np.empty_like(order)
    inv[order] = np.arange(prob.n)
    slots = inv[idx]
    ts = torch.tensor(slots, device=dev())
    ns = mesh.nsteps.cpu().numpy()[slots]
    assert np.array_equal(ns, om.nsteps)
    hs = mesh.h[:, ts].cpu().numpy().T
    assert mesh_rel_err(hs, om.h[:, :smax], ns) <= 1e-10
    mesh.h[:, ts] = tens(om.h[:, :smax].T.copy(), torch.float64)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    ti = torch.tensor(idx, device=dev())
    parity(gs.GradOut(out.loss[ti], out.dp[:, ti], out.du0[:, ti], None), sub, om)
