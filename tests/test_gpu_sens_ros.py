"""GPU <-> oracle parity for the forward sensitivities of the Rosenbrock
replays (gs_sens with ROS2 / ROS3): Robertson kinetics and Lorenz, the
matrices d u(t_k) / d (p, u0) against the oracle's dual numbers, the loss
gradient against the adjoint (gs_grad: the same derivative by reverse mode),
the loss bitwise equal to the replay's, fp32, and failed trajectories."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import TOL, ensemble, loss_args, mesh_from_oracle, parity

pytestmark = pytest.mark.gpu
EPS = np.finfo(np.float64).eps


def _prob(name, method, n):
    prob = W.by_name(name, n=n)
    prob.method = method
    if name == "lorenz_small":
        prob.rtol = prob.atol = 1e-5
    return prob


def _run(prob, om):
    ens = ensemble(prob)
    mesh = mesh_from_oracle(om, prob.dtype)
    out, S = gs.gs_sens(ens, mesh, **loss_args(prob))
    g = gs.gs_grad(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    return out, S.double().cpu().numpy(), g


@pytest.mark.parametrize("name,method", [("robertson", "ros2"), ("robertson", "ros3"), ("lorenz_small", "ros2"),
                                         ("lorenz_small", "ros3")])
def test_matches_oracle_and_adjoint(name, method):
    prob = _prob(name, method, 200)
    om = oracle.record(prob, 20000)
    assert (om.status == 0).all()
    out, S, g = _run(prob, om)
    ref = oracle.sens(prob, om)
    # per trajectory, largest entry error over the largest entry; the two
    # routes round differently at every step (eps per step)
    e = np.abs(S - ref).max(axis=(0, 1, 2)) / np.abs(ref).max(axis=(0, 1, 2))
    tol = max(1e-12, 8 * EPS * om.nsteps.max())
    assert e.max() <= tol, (e.max(), tol)
    # the gradient gate against the oracle (as for the adjoint: the stated
    # gate for 99 % of the trajectories, the worst within 4x the oracle's own
    # plain-precision routes)
    parity(out, prob, om)
    # forward mode = reverse mode (each within its own rounding of the exact
    # derivative), and the loss is the replay's, bit for bit
    assert torch.equal(out.loss, g.loss)
    for a, b in ((out.dp, g.dp), (out.du0, g.du0)):
        a, b = a.cpu().numpy(), b.cpu().numpy()
        assert (np.abs(a - b).max(0) / np.abs(b).max(0)).max() <= 4 * tol


def test_ros3_fp32():
    prob = _prob("lorenz_small", "ros3", 300)
    prob.dtype = "f32"
    prob.rtol = prob.atol = 1e-4
    om = oracle.record(prob, 8192)
    out, S, g = _run(prob, om)
    ref = oracle.sens(prob, om)
    e = np.abs(S - ref).max(axis=(0, 1, 2)) / np.abs(ref).max(axis=(0, 1, 2))
    assert e.max() <= TOL["f32"], e.max()
    parity(out, prob, om, tol=TOL["f32"])


def test_failed_and_ragged():
    """A failed trajectory gives NaN everywhere it owns; the rest are unchanged;
    n not a multiple of 128."""
    prob = _prob("robertson", "ros3", 131)
    om = oracle.record(prob, 20000)
    st = om.status.copy()
    st[7] = 1
    om_bad = oracle.Mesh(om.h, om.nsteps, om.save_idx, st, om.nreject)
    out, S, _ = _run(prob, om_bad)
    out0, S0, _ = _run(prob, om)
    assert np.isnan(S[..., 7]).all() and np.isnan(out.loss.cpu().numpy()[7])
    assert np.isnan(out.dp.cpu().numpy()[:, 7]).all() and np.isnan(out.du0.cpu().numpy()[:, 7]).all()
    keep = np.arange(prob.n) != 7
    assert np.array_equal(S[..., keep], S0[..., keep])


def test_full_size_sampled():
    """The 65,536-trajectory robertson ensemble with ROS3 in the benchmark's
    launch configuration; the oracle's dual numbers check a sample."""
    from gpu_util import dev
    prob = _prob("robertson", "ros3", None)
    ens = ensemble(prob)
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 20000)
    mesh = gs.new_mesh(prob.n, int(nsteps.max().item()), 1, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out, S = gs.gs_sens(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    assert (mesh.status == 0).all()
    from gpu_util import mesh_by_trajectory
    h, ns, si, st, order = mesh_by_trajectory(mesh)
    rng = np.random.default_rng(10)
    idx = np.unique(np.concatenate([rng.choice(prob.n, 64, replace=False), np.argsort(ns)[-8:]]))
    sub = prob.subset(idx)
    om = oracle.Mesh(h[idx].astype(np.float64), ns[idx], si[idx], st[idx], np.zeros(len(idx), np.int32))
    ref = oracle.sens(sub, om)
    got = S[..., torch.tensor(idx, device=dev())].double().cpu().numpy()
    e = np.abs(got - ref).max(axis=(0, 1, 2)) / np.abs(ref).max(axis=(0, 1, 2))
    assert e.max() <= max(1e-12, 8 * EPS * ns.max()), e.max()
