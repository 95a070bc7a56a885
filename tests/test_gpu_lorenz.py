"""GPU <-> oracle parity for the Tsit5 path on Lorenz (workloads lorenz_small
and lorenz_1m): recorder meshes (equal step counts, step sizes to 1e-10),
gradients on the same mesh (1e-12 fp64, 1e-4 fp32), forward-only solve."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import (TOL, dev, ensemble, grad_rel_err, loss_args, mesh_by_trajectory, mesh_from_oracle,
                      mesh_rel_err, parity, tens)

pytestmark = pytest.mark.gpu

def _record_gpu(prob, smax):
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, smax, len(prob.tsave), prob.dtype, dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    return ens, mesh


@pytest.fixture(scope="module")
def small():
    prob = W.lorenz_small()
    om = oracle.record(prob, 256)
    og = oracle.grad(prob, om)
    assert (om.status == 0).all()
    return prob, om, og


def test_record_matches_oracle(small):
    prob, om, og = small
    ens, mesh = _record_gpu(prob, 256)
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert (st == 0).all()
    assert np.array_equal(ns, om.nsteps)
    assert np.array_equal(si, om.save_idx)
    assert mesh_rel_err(h, om.h, ns) <= 1e-10
    # slots are ordered by decreasing step count
    nss = mesh.nsteps.cpu().numpy()
    assert (np.diff(nss) <= 0).all()
    assert np.array_equal(np.sort(order), np.arange(prob.n))


def test_count_matches_oracle(small):
    prob, om, og = small
    nsteps, status = gs.gs_count(ensemble(prob), prob.rtol, prob.atol, 256)
    torch.cuda.synchronize()
    assert np.array_equal(nsteps.cpu().numpy(), om.nsteps)
    assert (status.cpu().numpy() == 0).all()


@pytest.mark.parametrize("perm", [False, True])
def test_grad_on_oracle_mesh(small, perm):
    prob, om, og = small
    order = np.random.default_rng(2).permutation(prob.n) if perm else None
    out = gs.gs_grad(ensemble(prob), mesh_from_oracle(om, prob.dtype, order), **loss_args(prob))
    torch.cuda.synchronize()
    e = grad_rel_err(out, og)
    assert e.max() <= TOL["f64"], e.max()
    parity(out, prob, om)
    le = np.abs(out.loss.cpu().numpy() - og["loss"]) / np.abs(og["loss"])
    assert le.max() <= 1e-14, le.max()  # the forward replay follows the same contract


def test_grad_on_own_mesh(small):
    prob, om, og = small
    ens, mesh = _record_gpu(prob, 256)
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    same = np.array([np.array_equal(h[i], om.h[i]) for i in range(prob.n)])
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    e = grad_rel_err(out, og)
    assert same.mean() > 0.9
    assert e[same].max() <= TOL["f64"]


def test_solve_matches_oracle_replay(small):
    prob, om, og = small
    _, us = oracle.replay(prob, om)
    u = gs.gs_solve(ensemble(prob), mesh_from_oracle(om, prob.dtype)).cpu().numpy()
    assert np.abs(u - us).max() <= 1e-14 * np.abs(us).max()


@pytest.mark.parametrize("dtype,n", [("f64", 4000), ("f32", 2000)])
def test_lorenz_1m_shape(dtype, n):
    """Ten save points with targets, t in [0, 10]; n not a multiple of the block."""
    prob = W.lorenz_1m(n, dtype=dtype)
    om = oracle.record(prob, 1024)
    assert (om.status == 0).all()
    ens, mesh = _record_gpu(prob, 1024)
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    assert (st == 0).all()
    if dtype == "f64":
        assert np.array_equal(ns, om.nsteps)
        assert mesh_rel_err(h, om.h, ns) <= 1e-10
    else:
        # fp32 records follow the same contract in single precision
        assert np.array_equal(ns, om.nsteps)
        assert mesh_rel_err(h, om.h, ns) <= 1e-5
    out = gs.gs_grad(ens, mesh_from_oracle(om, dtype), **loss_args(prob))
    torch.cuda.synchronize()
    parity(out, prob, om)


@pytest.mark.parametrize("dtype", ["f64", "f32"])
def test_full_size_sampled(dtype):
    """2**20 trajectories in the launch configuration the benchmark times (the
    in-place re-record rewrites the whole mesh bit for bit); the oracle checks
    a sample (random + the longest chains) one by one.  fp64
    meshes equal the oracle's to 1e-10 (bitwise in practice); fp32 ones, of the
    fp32 instantiation of the oracle, have equal step counts on almost every
    trajectory and step sizes within fp32 rounding where they do."""
    prob = W.lorenz_1m(dtype=dtype)
    td = torch.float64 if dtype == "f64" else torch.float32
    ens = ensemble(prob)
    nsteps, status = gs.gs_count(ens, prob.rtol, prob.atol, 2048)
    ns_all = nsteps.cpu().numpy()
    rng = np.random.default_rng(11)
    idx = np.unique(np.concatenate([rng.choice(prob.n, 384, replace=False), np.argsort(ns_all)[-32:]]))
    sub = prob.subset(idx)
    om = oracle.record(sub, 2048)
    assert (om.status == 0).all()
    smax = max(int(nsteps.max().item()), int(om.nsteps.max()))
    mesh = gs.new_mesh(prob.n, smax, 10, dtype, dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    assert (mesh.status == 0).all()
    # the benchmark's steps re-record in place: the whole mesh, bit for bit
    ref = [t.clone() for t in (mesh.h, mesh.order, mesh.nsteps, mesh.save_idx, mesh.status, mesh.nreject)]
    gs.gs_record_inplace(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    for a, b in zip(ref, (mesh.h, mesh.order, mesh.nsteps, mesh.save_idx, mesh.status, mesh.nreject)):
        assert torch.equal(a, b)
    del ref
    # mesh parity on the sample
    order = mesh.order.cpu().numpy()
    inv = np.empty_like(order)
    inv[order] = np.arange(prob.n)
    slots = inv[idx]
    hs = mesh.h[:, torch.tensor(slots, device=dev())].double().cpu().numpy().T
    ns = mesh.nsteps.cpu().numpy()[slots]
    if dtype == "f64":
        assert np.array_equal(ns, om.nsteps)
        assert mesh_rel_err(hs, om.h[:, :smax], ns) <= 1e-10
    else:
        same = ns == om.nsteps
        assert same.mean() >= 0.97, same.mean()
        assert mesh_rel_err(hs[same], om.h[same, :smax], ns[same]) <= 1e-5
    # gradient parity on the oracle's mesh, injected into the sampled slots of
    # the full-size mesh (trajectories are independent)
    ts = torch.tensor(slots, device=dev())
    hi = np.zeros((smax, len(idx)))
    hi[:] = om.h[:, :smax].T
    mesh.h[:, ts] = tens(hi, td)
    mesh.nsteps[ts] = tens(om.nsteps.astype(np.int32), torch.int32)
    mesh.save_idx[:, ts] = tens(om.save_idx.T.astype(np.int32), torch.int32)
    out = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    ti = torch.tensor(idx, device=dev())
    sub_out = gs.GradOut(out.loss[ti], out.dp[:, ti], out.du0[:, ti], None)
    parity(sub_out, sub, om)
    assert torch.isfinite(out.dp).all() and torch.isfinite(out.du0).all()
