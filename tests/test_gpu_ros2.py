"""GPU <-> oracle parity for the Rosenbrock (ROS2) path: Robertson kinetics
(workload robertson, linear loss) and Lorenz integrated with ROS2."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import dev, ensemble, grad_rel_err, loss_args, mesh_by_trajectory, mesh_from_oracle, mesh_rel_err, parity, tens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rob():
    prob = W.robertson(300)
    om = oracle.record(prob, 16384)
    og = oracle.grad(prob, om)
    assert (om.status == 0).all()
    return prob, om, og


def test_robertson_record(rob):
    prob, om, og = rob
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 16384, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert (st == 0).all()
    assert np.array_equal(ns, om.nsteps)
    assert mesh_rel_err(h, om.h, ns) <= 1e-10


def test_robertson_grad(rob):
    prob, om, og = rob
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    e = grad_rel_err(out, og)
    assert e.max() <= 1e-12, e.max()
    assert np.abs(out.loss.cpu().numpy() - og["loss"]).max() <= 1e-14 * np.abs(og["loss"]).max()


def test_robertson_solve(rob):
    prob, om, og = rob
    _, us = oracle.replay(prob, om)
    u = gs.gs_solve(ensemble(prob), mesh_from_oracle(om, "f64")).cpu().numpy()
    assert np.abs(u - us).max() <= 1e-14


def test_lorenz_ros2_grad():
    prob = W.lorenz_small(500)
    prob.method = "ros2"
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
    out = gs.gs_grad(ens, mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    assert grad_rel_err(out, og).max() <= 1e-12


def test_robertson_full_size_sampled():
    prob = W.robertson()
    ens = ensemble(prob)
    nsteps, status = gs.gs_count(ens, prob.rtol, prob.atol, 20000)
    smax = int(nsteps.max().item())
    mesh = gs.new_mesh(prob.n, smax, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    assert (mesh.status == 0).all()
    rng = np.random.default_rng(5)
    idx = np.sort(rng.choice(prob.n, 96, replace=False))
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
