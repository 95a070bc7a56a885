"""Edge cases of the GPU path: tiny and ragged ensembles, failing
trajectories, invariances, call errors."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import dev, ensemble, grad_rel_err, loss_args, mesh_by_trajectory, mesh_from_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [1, 31, 129])
def test_tiny_and_ragged(n):
    prob = W.lorenz_small(n)
    om = oracle.record(prob, 256)
    og = oracle.grad(prob, om)
    ens = ensemble(prob)
    mesh = gs.new_mesh(n, 256, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert np.array_equal(ns, om.nsteps)
    assert grad_rel_err(out, og).max() <= 1e-12


def test_capacity_and_nonfinite_statuses():
    prob = W.lorenz_small(64)
    prob.p = prob.p.copy()
    prob.p[0, 5] = np.nan
    om = oracle.record(prob, 140)  # some trajectories need more than 140 steps
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 140, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    u = gs.gs_solve(ens, mesh)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert np.array_equal(st, om.status)
    assert st[5] == gs.gradsolve.TRAJ_NONFINITE and (st == gs.gradsolve.TRAJ_MAXSTEPS).any()
    bad = st != 0
    assert torch.isnan(out.loss.cpu()[torch.tensor(bad)]).all()
    assert torch.isfinite(out.dp.cpu()[:, torch.tensor(~bad)]).all()
    assert torch.isnan(u.cpu()[:, :, torch.tensor(bad)]).all()


def test_leading_zero_steps_are_identities():
    prob = W.lorenz_small(100)
    om = oracle.record(prob, 256)
    ens = ensemble(prob)
    ref = gs.gs_grad(ens, mesh_from_oracle(om, "f64"), **loss_args(prob))
    z = 5
    om2 = oracle.Mesh(np.concatenate([np.zeros((prob.n, z)), om.h], 1), om.nsteps + z, om.save_idx + z,
                      om.status, om.nreject)
    out = gs.gs_grad(ens, mesh_from_oracle(om2, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    for a, b in ((out.loss, ref.loss), (out.dp, ref.dp), (out.du0, ref.du0)):
        assert torch.equal(a, b)


def test_permuted_slots_give_identical_bits():
    prob = W.lorenz_1m(300)
    om = oracle.record(prob, 1024)
    ens = ensemble(prob)
    a = gs.gs_grad(ens, mesh_from_oracle(om, "f64"), **loss_args(prob))
    b = gs.gs_grad(ens, mesh_from_oracle(om, "f64", np.random.default_rng(0).permutation(prob.n)),
                   **loss_args(prob))
    torch.cuda.synchronize()
    assert torch.equal(a.dp, b.dp) and torch.equal(a.du0, b.du0) and torch.equal(a.loss, b.loss)


def test_call_errors():
    prob = W.lorenz_small(16)
    ens = ensemble(prob)
    mesh = gs.new_mesh(16, 256, 1, "f64", dev())
    with pytest.raises(gs.gradsolve.GradsolveError) as e:
        gs.gs_grad(ens, mesh, ws=gs.workspace(16, dev()))
    assert e.value.code == gs.gradsolve.GS_EWORKSPACE
    big = gs.new_mesh(16, 256, 3, "f64", dev())
    with pytest.raises(gs.gradsolve.GradsolveError):
        gs.gs_solve(ens, big)
    ens_rt = ensemble(W.robertson(16))
    ens_rt.method = "tsit5"
    with pytest.raises(gs.gradsolve.GradsolveError) as e:
        gs.gs_grad(ens_rt, gs.new_mesh(16, 64, 1, "f64", dev()), loss="linear",
                   weight=torch.ones((1, 3, 16), dtype=torch.float64, device=dev()))
    assert e.value.code == gs.gradsolve.GS_EUNSUPPORTED


def test_ros3_statuses_and_nan_outputs():
    """ROS3 on Robertson: a NaN rate constant gives NONFINITE, a capacity below
    some trajectories' step counts gives MAXSTEPS, both as the oracle's; the
    failed trajectories get NaN from the gradient, the replay and the
    sensitivities, the others finite values."""
    prob = W.robertson(64)
    prob.method = "ros3"
    prob.p = prob.p.copy()
    prob.p[2, 5] = np.nan
    full = oracle.record(prob, 20000)
    smax = int(np.median(full.nsteps[full.status == 0]))
    om = oracle.record(prob, smax)
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, smax, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    u = gs.gs_solve(ens, mesh)
    so, S = gs.gs_sens(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert np.array_equal(st, om.status)
    assert st[5] == gs.gradsolve.TRAJ_NONFINITE and (st == gs.gradsolve.TRAJ_MAXSTEPS).any() and (st == 0).any()
    bad = torch.tensor(st != 0)
    for t in (out.loss.cpu(), so.loss.cpu()):
        assert torch.isnan(t[bad]).all() and torch.isfinite(t[~bad]).all()
    assert torch.isnan(out.dp.cpu()[:, bad]).all() and torch.isfinite(out.dp.cpu()[:, ~bad]).all()
    assert torch.isnan(u.cpu()[:, :, bad]).all() and torch.isfinite(u.cpu()[:, :, ~bad]).all()
    assert torch.isnan(S.cpu()[..., bad]).all() and torch.isfinite(S.cpu()[..., ~bad]).all()


def test_ros3_leading_zero_steps_are_identities():
    prob = W.robertson(40)
    prob.method = "ros3"
    om = oracle.record(prob, 20000)
    ens = ensemble(prob)
    ref = gs.gs_grad(ens, mesh_from_oracle(om, "f64"), **loss_args(prob))
    z = 3
    om2 = oracle.Mesh(np.concatenate([np.zeros((prob.n, z)), om.h], 1), om.nsteps + z, om.save_idx + z,
                      om.status, om.nreject)
    out = gs.gs_grad(ens, mesh_from_oracle(om2, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    for a, b in ((out.loss, ref.loss), (out.dp, ref.dp), (out.du0, ref.du0)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("n", [1, 129])
def test_node64_tensor_cores_tiny_ragged_and_nonfinite(n):
    """The 128-trajectory tensor-core recorder and gradient with a CTA that is
    nearly empty (n = 1) or ragged (n = 129), one trajectory with a NaN input:
    NONFINITE for it alone, the rest within the fp32 gate of the oracle."""
    from gpu_util import parity
    prob = W.node64(n)
    prob.u0 = prob.u0.copy()
    prob.u0[3, n - 1] = np.nan
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 64, 1, "f32", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert st[n - 1] == gs.gradsolve.TRAJ_NONFINITE and (st[: n - 1] == 0).all()
    assert torch.isnan(out.loss.cpu()[n - 1]) and torch.isnan(out.dp.cpu()[:, n - 1]).all()
    assert torch.isfinite(out.dshared).all()
    if n > 1:
        idx = np.arange(n - 1)
        sub = prob.subset(idx)
        om = oracle.Mesh(h[idx].astype(np.float64), ns[idx], si[idx], st[idx], np.zeros(len(idx), np.int32))
        ti = torch.tensor(idx, device=dev())
        parity(gs.GradOut(out.loss[ti], out.dp[:, ti], out.du0[:, ti], None), sub, om, dual=False)
