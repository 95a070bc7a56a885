"""GPU <-> oracle parity for Verner's 7(6) pair on Lorenz: the record (step
counts, step sizes, save indices: bitwise in fp64), the sizing pass, the
replay and the adaptive forward-only solve (bitwise), the fused gradient
(fp64 and fp32, per-trajectory gate) on the oracle's mesh in any slot order
and on the GPU's own record, the in-place re-record, the forward
sensitivities (matrices against the oracle's, gradient equal to the
adjoint's), and the 2**20 ensemble of the benchmark in its launch
configuration on a sample."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import (TOL, dev, ensemble, loss_args, mesh_by_trajectory, mesh_from_oracle, parity, sens_parity)

pytestmark = pytest.mark.gpu


def _prob(n, dtype="f64", name="lorenz_1m"):
    prob = W.by_name(name, n=n, dtype=dtype) if name == "lorenz_1m" else W.by_name(name, n=n)
    return dataclasses.replace(prob, method="vern7")


@pytest.fixture(scope="module")
def case():
    prob = _prob(2000)
    om = oracle.record(prob, 1024)
    assert (om.status == 0).all()
    return prob, om


def test_record_matches_oracle(case):
    prob, om = case
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 1024, len(prob.tsave), "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert (st == 0).all()
    assert np.array_equal(ns, om.nsteps) and np.array_equal(si, om.save_idx)
    for i in range(prob.n):
        assert np.array_equal(h[i, : ns[i]], om.h[i, : ns[i]]), i  # the same arithmetic: bitwise
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 1024)
    torch.cuda.synchronize()
    assert np.array_equal(nsteps.cpu().numpy(), om.nsteps)
    # re-recording in place keeps the slot order and gives the same mesh
    before = mesh.order.clone()
    gs.gs_record_inplace(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    assert torch.equal(before, mesh.order)
    h2, ns2, si2, st2, _ = mesh_by_trajectory(mesh)
    assert np.array_equal(h2, h) and np.array_equal(ns2, ns) and np.array_equal(si2, si)


def test_replay_and_adaptive_solve(case):
    prob, om = case
    _, us = oracle.replay(prob, om)
    u = gs.gs_solve(ensemble(prob), mesh_from_oracle(om, "f64")).cpu().numpy()
    assert np.array_equal(u, us)
    ua, na, sa = gs.gs_solve_adaptive(ensemble(prob), prob.rtol, prob.atol, 1024)
    torch.cuda.synchronize()
    uo, no, so = oracle.solve_adaptive(prob, 1024)
    assert (sa.cpu().numpy() == 0).all() and np.array_equal(na.cpu().numpy(), no)
    assert np.array_equal(ua.cpu().numpy(), uo)


@pytest.mark.parametrize("perm", [False, True])
def test_gradient_on_oracle_mesh(case, perm):
    prob, om = case
    order = np.random.default_rng(5).permutation(prob.n) if perm else None
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f64", order), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om)
    loss, _ = oracle.replay(prob, om)
    assert np.abs(out.loss.cpu().numpy() - loss).max() <= 1e-14 * np.abs(loss).max()


def test_gradient_short_horizon_meets_the_stated_gate():
    """Lorenz on t in [0, 1] (well conditioned): every trajectory within
    1e-12 of the oracle, no allowance."""
    prob = _prob(1000, name="lorenz_small")
    om = oracle.record(prob, 512)
    assert (om.status == 0).all()
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f64"), **loss_args(prob))
    torch.cuda.synchronize()
    e = parity(out, prob, om, c=0.0)
    assert e.max() <= 1e-12, e.max()


def test_gradient_fp32():
    prob = _prob(1000, dtype="f32")
    om = oracle.record(prob, 1024)
    assert (om.status == 0).all()
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, "f32"), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om)


def test_gradient_on_own_record_and_linear_loss():
    prob = _prob(700, name="lorenz_small")
    w = np.random.default_rng(11).uniform(-1.0, 1.0, (1, 3, prob.n))
    prob = dataclasses.replace(prob, loss="linear", weight=w, target=None)
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 512, 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    h, ns, si, st, _ = mesh_by_trajectory(mesh)
    om = oracle.Mesh(h, ns, si, st, np.zeros(prob.n, np.int32))
    parity(out, prob, om)


@pytest.mark.parametrize("dtype", ["f64", "f32"])
def test_forward_sensitivities(dtype):
    """d u(t_k)/d(p, u0) at the ten save points of the headline ensemble's
    first trajectories, against the oracle's wide-tape matrices with the
    per-trajectory gate; the loss bitwise that of the oracle's replay (fp64),
    the gradient equal to the oracle's."""
    prob = _prob(256, dtype=dtype)
    om = oracle.record(prob, 1024)
    assert (om.status == 0).all()
    out, S = gs.gs_sens(ensemble(prob), mesh_from_oracle(om, dtype), **loss_args(prob))
    torch.cuda.synchronize()
    sens_parity(S.double().cpu().numpy(), prob, om, TOL[dtype])
    parity(out, prob, om)
    if dtype == "f64":
        loss, _ = oracle.replay(prob, om)
        assert np.array_equal(out.loss.cpu().numpy(), loss)


def test_failed_trajectories_are_nan(case):
    """Slots whose status is not OK (or whose step count is out of range) get
    NaN loss, gradient and sensitivities; the others are unaffected."""
    prob, om = case
    sub = prob.subset(np.arange(8))
    st = np.zeros(8, np.int32)
    st[[1, 5]] = 2  # GS_TRAJ_DTMIN
    ns = om.nsteps[:8].copy()
    ns[6] = om.h.shape[1] + 1  # beyond the mesh capacity
    bad = oracle.Mesh(om.h[:8], ns, om.save_idx[:8], st, om.nreject[:8])
    good = oracle.Mesh(om.h[:8], om.nsteps[:8], om.save_idx[:8], np.zeros(8, np.int32), om.nreject[:8])
    ens = ensemble(sub)
    out = gs.gs_grad(ens, mesh_from_oracle(bad, "f64"), **loss_args(sub))
    ref = gs.gs_grad(ens, mesh_from_oracle(good, "f64"), **loss_args(sub))
    sens_out, S = gs.gs_sens(ens, mesh_from_oracle(bad, "f64"), **loss_args(sub))
    torch.cuda.synchronize()
    failed = np.array([1, 5, 6])
    ok = np.setdiff1d(np.arange(8), failed)
    for o in (out, sens_out):
        for t in (o.loss.cpu().numpy()[None, :], o.dp.cpu().numpy(), o.du0.cpu().numpy()):
            assert np.isnan(t[:, failed]).all() and np.isfinite(t[:, ok]).all()
    assert np.isnan(S.cpu().numpy()[..., failed]).all()
    assert np.array_equal(out.dp.cpu().numpy()[:, ok], ref.dp.cpu().numpy()[:, ok])


def test_unsupported_paths():
    prob = _prob(4)
    ens = ensemble(prob)
    with pytest.raises(gs.gradsolve.GradsolveError):  # Verner records land on the save times
        gs.gs_count(ens, prob.rtol, prob.atol, 100, dense=True)
    mesh = gs.new_mesh(prob.n, 512, len(prob.tsave), "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    rob = dataclasses.replace(W.robertson(4), method="vern7")
    rmesh = gs.new_mesh(rob.n, 64, 1, "f64", dev())
    with pytest.raises(gs.gradsolve.GradsolveError):  # the gradient is built for Lorenz
        gs.gs_grad(ensemble(rob), rmesh, **loss_args(rob))
    with pytest.raises(gs.gradsolve.GradsolveError):  # and so are the forward sensitivities
        gs.gs_sens(ensemble(rob), rmesh, **loss_args(rob))


def test_full_size_sampled():
    """The 2**20 ensemble recorded and differentiated in the benchmark's
    launch configuration; the oracle checks a sample (random slots and the
    longest chains) on the GPU's own mesh."""
    prob = _prob(1 << 20)
    ens = ensemble(prob)
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 4096)
    smax = int(nsteps.max())
    mesh = gs.new_mesh(prob.n, smax, len(prob.tsave), "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    order = mesh.order.cpu().numpy()
    rng = np.random.default_rng(13)
    slots = np.concatenate([np.arange(64), rng.choice(prob.n, 448, replace=False)])
    idx = order[slots]
    sub = prob.subset(idx)
    ns = mesh.nsteps.cpu().numpy()[slots]
    h = mesh.h[:, torch.as_tensor(slots, device=mesh.h.device)].double().cpu().numpy().T
    si = mesh.save_idx[:, torch.as_tensor(slots, device=mesh.h.device)].cpu().numpy().T
    st = mesh.status.cpu().numpy()[slots]
    assert (st == 0).all()
    om = oracle.Mesh(h, ns, si, st, np.zeros(len(idx), np.int32))
    # the sampled meshes equal the oracle's own record of those trajectories
    orec = oracle.record(sub, smax)
    assert np.array_equal(orec.nsteps, ns) and np.array_equal(orec.h[:, :smax], h)

    class Sub:
        dp = out.dp[:, torch.as_tensor(idx, device=out.dp.device)]
        du0 = out.du0[:, torch.as_tensor(idx, device=out.dp.device)]
    parity(Sub, sub, om)
